// k2_gemm_i8.cu -- forward int8 GEMM of the int8-LoRA Dense layer on the
// 5th-generation tensor cores, with the whole layer epilogue fused:
//
//   acc[m,n] = sum_k Xq[m,k] Wq[n,k]                    (int32, in TMEM)
//   Y[m,n]   = acc * sx[m] * sw[n] + bias[n] + c * sum_j xA[m,j] B[j,n]
//
// ("Introduce QLoRA-like technique", Results: int8 Dense needs a hardware
// int8 matmul; "Parameter-efficient fine-tuning of GPT-2 with LoRA", "LoRA
// equation" for the added low-rank term, with xA = x . A from the input pass.)
//
// Persistent kernel, one CTA per SM, 10 warps:
//   warp 0      TMA producer: Xq [128 x 128] and Wq [BN x 128] int8 tiles
//               (128B swizzle, K-major) into a STAGES-deep ring
//   warp 1      TMEM owner and MMA issuer: tcgen05.mma.kind::i8, M=128,
//               N=BN, K=32, into one of two TMEM accumulators (2 x BN
//               columns), so that tile i+1's main loop overlaps tile i's
//               epilogue
//   warps 2..9  epilogue: two warps per TMEM lane quarter, each one half of
//               the columns; scale, bias and the rank-r term per element,
//               then a staged, coalesced 16-byte store of the output block
// Ragged M, N, K: the tensor maps zero-fill, the stores are predicated.
#include "internal.h"
#include "ptx.cuh"
#include "tile_epilogue.cuh"

namespace qlora {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 128;  // int8 elements per k-block: one 128-byte swizzle row
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kSmemLimit = 232448;  // 227 KB opt-in dynamic shared memory

template <int BN, typename OutT, int RMAX>
struct K2Cfg {
    static constexpr int kRPad = RMAX <= 16 ? ((RMAX + 3) / 4) * 4 : 0;  // B table width
    static constexpr int kABytes = kBM * kBK;
    static constexpr int kBBytes = BN * kBK;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStgBytes = kEpiWarps * 32 * stage_pitch<OutT>();
    static constexpr int kParamBytes = BN * 4 * 2 + BN * kRPad * 4;
    static constexpr int kFixed = kStgBytes + kParamBytes + 256 + 1024;
    static constexpr int kStagesFit = (kSmemLimit - kFixed) / kStageBytes;
    static constexpr int STAGES = kStagesFit > 8 ? 8 : kStagesFit;
    static_assert(STAGES >= 2, "shared memory budget");
    static constexpr int kStgOff = STAGES * kStageBytes;
    static constexpr int kSwOff = kStgOff + kStgBytes;
    static constexpr int kBiasOff = kSwOff + BN * 4;
    static constexpr int kTabOff = kBiasOff + BN * 4;
    static constexpr int kBarOff = kTabOff + BN * kRPad * 4;
    static constexpr int kTotal = kBarOff + 256 + 1024;
    static constexpr uint32_t kTmemCols = 2 * BN;
};

template <int BN, typename OutT, int RMAX>
__global__ void __launch_bounds__(kThreads, 1)
    k2_gemm_i8_lora_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB, int M, int N, int K,
                           FwdEpilogue ep, int* status) {
    using C = K2Cfg<BN, OutT, RMAX>;
    constexpr int S = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;   // [2]
    uint64_t* tempty = tfull + 2;  // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    float* s_sw = reinterpret_cast<float*>(smem + C::kSwOff);
    float* s_bias = reinterpret_cast<float*>(smem + C::kBiasOff);
    float* s_tab = reinterpret_cast<float*>(smem + C::kTabOff);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int num_n = (N + BN - 1) / BN;
    const int tiles = ((M + kBM - 1) / kBM) * num_n;
    const int nkb = (K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kEpiWarps);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            int g = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int m0 = (t / num_n) * kBM;
                const int n0 = (t % num_n) * BN;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % S;
                    if (g >= S && !mbar_wait(&empty[s], ((g / S) - 1) & 1, status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + s * C::kStageBytes;
                    mbar_arrive_expect_tx(&full[s], C::kStageBytes);
                    tma_load_2d(sa, &tmA, &full[s], kb * kBK, m0);
                    tma_load_2d(sa + C::kABytes, &tmB, &full[s], kb * kBK, n0);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kBM, BN);
            int g = 0, i = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++i) {
                const int ab = i & 1;
                const int use = i >> 1;
                if (use > 0 && !mbar_wait(&tempty[ab], (use - 1) & 1, status)) break;
                tc_fence_after();
                const uint32_t dacc = tmem + ab * BN;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % S;
                    if (!mbar_wait(&full[s], (g / S) & 1, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + s * C::kStageBytes);
                    const uint32_t b_base = a_base + C::kABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 32; ++kk) {
                        const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024, kLayoutSw128);
                        const uint64_t bd = smem_desc(b_base + kk * 32, 16, 1024, kLayoutSw128);
                        mma_i8(dacc, ad, bd, idesc, (kb | kk) != 0);
                    }
                    mma_commit(&empty[s]);
                }
                if (ok) mma_commit(&tfull[ab]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int ew = warp - 2;            // 0 .. 7
        const int q = warp & 3;             // TMEM lane quarter of this warp
        const int half = ew >> 2;           // column half
        const int et = threadIdx.x - 64;    // 0 .. 255
        uint8_t* stg = smem + C::kStgOff + ew * 32 * stage_pitch<OutT>();
        const bool vec = ((static_cast<size_t>(N) * sizeof(OutT)) % 16) == 0;
        OutT* Y = static_cast<OutT*>(ep.Y);
        int i = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
            const int ab = i & 1;
            const int use = i >> 1;
            const int m0 = (t / num_n) * kBM;
            const int n0 = (t % num_n) * BN;
            // per-column tables of this tile (after every warp is done with the last ones)
            named_bar_sync(1, 32 * kEpiWarps);
            for (int c = et; c < BN; c += 32 * kEpiWarps) {
                const int n = n0 + c;
                s_sw[c] = n < N ? ep.sw[n] : 0.f;
                s_bias[c] = (n < N && ep.bias) ? ep.bias[n] : 0.f;
            }
            if constexpr (C::kRPad > 0) {
                for (int e = et; e < BN * C::kRPad; e += 32 * kEpiWarps) {
                    const int c = e / C::kRPad, j = e % C::kRPad;
                    const int n = n0 + c;
                    s_tab[e] = (n < N && j < ep.r) ? ep.B[static_cast<size_t>(j) * N + n] : 0.f;
                }
            }
            named_bar_sync(1, 32 * kEpiWarps);

            const int row0 = m0 + q * 32;
            const int row = row0 + lane;
            const bool row_ok = row < M;
            const float sxm = row_ok ? ep.sx[row] : 0.f;
            float xa[RMAX];
#pragma unroll
            for (int j = 0; j < RMAX; ++j)
                xa[j] = (row_ok && j < ep.r) ? ep.xA[static_cast<size_t>(row) * ep.r + j] * ep.c : 0.f;

            const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[ab], use & 1, status));
            if (!ok) break;
            tc_fence_after();
            const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + ab * BN;
#pragma unroll 1
            for (int col = half * (BN / 2); col < (half + 1) * (BN / 2); col += kEpiCols) {
                uint32_t v[kEpiCols];
                tmem_ld16(tbase + col, v);
                tmem_ld_wait();
                float y[kEpiCols];
#pragma unroll
                for (int e = 0; e < kEpiCols; ++e) {
                    const int c = col + e;
                    const float a = static_cast<float>(static_cast<int32_t>(v[e]));
                    float acc = fmaf(a * sxm, s_sw[c], s_bias[c]);
                    if constexpr (C::kRPad > 0) {
                        const float4* tb = reinterpret_cast<const float4*>(s_tab + c * C::kRPad);
#pragma unroll
                        for (int j4 = 0; j4 < C::kRPad / 4; ++j4) {
                            const float4 b4 = tb[j4];
                            acc = fmaf(xa[4 * j4], b4.x, acc);
                            if (4 * j4 + 1 < RMAX) acc = fmaf(xa[4 * j4 + 1], b4.y, acc);
                            if (4 * j4 + 2 < RMAX) acc = fmaf(xa[4 * j4 + 2], b4.z, acc);
                            if (4 * j4 + 3 < RMAX) acc = fmaf(xa[4 * j4 + 3], b4.w, acc);
                        }
                    } else {
                        const int n = n0 + c;
                        if (n < N)
                            for (int j = 0; j < ep.r; ++j)
                                acc = fmaf(xa[j], __ldg(ep.B + static_cast<size_t>(j) * N + n), acc);
                    }
                    y[e] = acc;
                }
                if (ep.acc && row_ok) {
                    for (int e = 0; e < kEpiCols; ++e)
                        if (n0 + col + e < N)
                            ep.acc[static_cast<size_t>(row) * N + n0 + col + e] = static_cast<int32_t>(v[e]);
                }
                store_block<OutT>(stg, y, lane, Y, static_cast<size_t>(N), row0, M, n0 + col, N, vec);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[ab]);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int BN, typename OutT, int RMAX>
cudaError_t launch_cfg(const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K,
                       const FwdEpilogue& ep, int* status, cudaStream_t s) {
    using C = K2Cfg<BN, OutT, RMAX>;
    auto kern = k2_gemm_i8_lora_kernel<BN, OutT, RMAX>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), C::kTotal);
    if (e != cudaSuccess) return e;
    const int tiles = ((M + kBM - 1) / kBM) * ((N + BN - 1) / BN);
    const int grid = tiles < sm_count() ? tiles : sm_count();
    kern<<<grid, kThreads, C::kTotal, s>>>(ta, tb, M, N, K, ep, status);
    return cudaGetLastError();
}

template <typename OutT, int RMAX>
cudaError_t launch_bn(int bn, const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K,
                      const FwdEpilogue& ep, int* status, cudaStream_t s) {
    if (bn == 256) return launch_cfg<256, OutT, RMAX>(ta, tb, M, N, K, ep, status, s);
    if (bn == 128) return launch_cfg<128, OutT, RMAX>(ta, tb, M, N, K, ep, status, s);
    return launch_cfg<64, OutT, RMAX>(ta, tb, M, N, K, ep, status, s);
}

template <typename OutT>
cudaError_t launch_r(int bn, const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K,
                     const FwdEpilogue& ep, int* status, cudaStream_t s) {
    if (ep.r <= 4) return launch_bn<OutT, 4>(bn, ta, tb, M, N, K, ep, status, s);
    if (ep.r <= 8) return launch_bn<OutT, 8>(bn, ta, tb, M, N, K, ep, status, s);
    if (ep.r <= 16) return launch_bn<OutT, 16>(bn, ta, tb, M, N, K, ep, status, s);
    return launch_bn<OutT, 64>(bn, ta, tb, M, N, K, ep, status, s);
}

}  // namespace

cudaError_t launch_gemm_i8_fwd(Act act, const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                               const FwdEpilogue& ep, int* status, cudaStream_t s) {
    // Tile width: the widest BN that still gives every SM a tile.
    const int mt = (M + kBM - 1) / kBM;
    const int sms = sm_count();
    int bn = 256;
    while (bn > 64 && mt * ((N + bn - 1) / bn) < sms) bn /= 2;
    CUtensorMap ta, tb;
    if (!make_tmap_2d(&ta, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K, K, kBM, kBK,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_tmap_2d(&tb, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, K, bn, kBK,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (act == kBF16) return launch_r<__nv_bfloat16>(bn, ta, tb, M, N, K, ep, status, s);
    return launch_r<float>(bn, ta, tb, M, N, K, ep, status, s);
}

}  // namespace qlora
