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
// Structure (one 128 x BN output tile per CTA, 6 warps):
//   warp 0      TMA producer: Xq and Wq tiles (128-byte rows, 128B swizzle)
//               into a STAGES-deep shared-memory ring, one mbarrier per stage
//   warp 1      allocates BN TMEM columns and issues tcgen05.mma.kind::i8
//               (M=128, N=BN, K=32 per instruction) from one thread, then
//               tcgen05.commit to release each stage and finally the tile
//   warps 2..5  epilogue: tcgen05.ld of their 32 TMEM lanes, scale, bias and
//               the rank-r LoRA term, predicated stores of Y
// Both operands are K-major (Xq rows and Wq rows are contiguous in K).
// The tensor maps zero-fill out-of-range rows/columns, so ragged M, N, K need
// no special path; the epilogue predicates its stores.
#include "internal.h"
#include "ptx.cuh"

namespace qlora {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 128;  // int8 elements per k-block: one 128-byte swizzle row
constexpr int kThreads = 192;

template <int BN, int STAGES>
struct K2Layout {
    static constexpr int kABytes = kBM * kBK;
    static constexpr int kBBytes = BN * kBK;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kBarOff = STAGES * kStageBytes;
    static constexpr int kSwOff = kBarOff + 256;             // sw tile  [BN]
    static constexpr int kBiasOff = kSwOff + BN * 4;         // bias tile [BN]
    static constexpr int kLoraOff = kBiasOff + BN * 4;       // B tile [16][BN] (r <= 16)
    static constexpr int kTotal = kLoraOff + 16 * BN * 4 + 1024;  // + alignment slack
};

template <typename OutT>
__device__ __forceinline__ void store_out(OutT* p, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* p, float v) {
    *p = __float2bfloat16_rn(v);
}

template <int BN, int STAGES, typename OutT, int RMAX>
__global__ void __launch_bounds__(kThreads, 1)
    k2_gemm_i8_lora_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB, int M, int N, int K,
                           FwdEpilogue ep, int* status) {
    using L = K2Layout<BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 1);
    float* s_sw = reinterpret_cast<float*>(smem + L::kSwOff);
    float* s_bias = reinterpret_cast<float*>(smem + L::kBiasOff);
    float* s_lb = reinterpret_cast<float*>(smem + L::kLoraOff);
    constexpr bool kStageB = RMAX <= 16;

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int m0 = blockIdx.y * kBM;
    const int n0 = blockIdx.x * BN;
    const int nkb = (K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, BN);
        tmem_relinquish();
    }
    // per-channel vectors of this tile, staged once for the epilogue
    for (int i = threadIdx.x; i < BN; i += kThreads) {
        const int n = n0 + i;
        s_sw[i] = n < N ? ep.sw[n] : 0.f;
        s_bias[i] = (n < N && ep.bias) ? ep.bias[n] : 0.f;
    }
    if constexpr (kStageB) {
        for (int i = threadIdx.x; i < RMAX * BN; i += kThreads) {
            const int j = i / BN, n = n0 + i % BN;
            s_lb[i] = (j < ep.r && n < N) ? ep.B[static_cast<size_t>(j) * N + n] : 0.f;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % STAGES;
                const int it = kb / STAGES;
                if (kb >= STAGES && !mbar_wait(&empty[s], (it - 1) & 1, status)) break;
                uint8_t* sa = smem + s * L::kStageBytes;
                uint8_t* sb = sa + L::kABytes;
                mbar_arrive_expect_tx(&full[s], L::kStageBytes);
                tma_load_2d(sa, &tmA, &full[s], kb * kBK, m0);
                tma_load_2d(sb, &tmB, &full[s], kb * kBK, n0);
            }
        }
        __syncwarp();  // reconverge the warp before the teardown barrier
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kBM, BN);
            bool ok = true;
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % STAGES;
                const int it = kb / STAGES;
                if (!mbar_wait(&full[s], it & 1, status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a_base = smem_u32(smem + s * L::kStageBytes);
                const uint32_t b_base = a_base + L::kABytes;
#pragma unroll
                for (int kk = 0; kk < kBK / 32; ++kk) {
                    const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024, kLayoutSw128);
                    const uint64_t bd = smem_desc(b_base + kk * 32, 16, 1024, kLayoutSw128);
                    mma_i8(tmem, ad, bd, idesc, (kb | kk) != 0);
                }
                mma_commit(&empty[s]);
            }
            if (ok) mma_commit(tfull);
        }
        __syncwarp();  // reconverge the warp before the teardown barrier
    } else {
        // epilogue: warps 2..5 -> TMEM lane quarters 2,3,0,1
        const int q = warp & 3;
        const int row = m0 + q * 32 + lane;
        const bool row_ok = row < M;
        float sxm = 0.f;
        float xa[RMAX];
#pragma unroll
        for (int j = 0; j < RMAX; ++j)
            xa[j] = (row_ok && j < ep.r) ? ep.xA[static_cast<size_t>(row) * ep.r + j] * ep.c : 0.f;
        if (row_ok) sxm = ep.sx[row];
        // warp-uniform, so that the .sync.aligned TMEM loads below stay converged
        const bool ok = __all_sync(0xffffffffu, mbar_wait(tfull, 0, status));
        tc_fence_after();
        if (ok) {
            OutT* yrow = static_cast<OutT*>(ep.Y) + static_cast<size_t>(row_ok ? row : 0) * N;
            int32_t* arow = ep.acc ? ep.acc + static_cast<size_t>(row_ok ? row : 0) * N : nullptr;
#pragma unroll 1
            for (int col = 0; col < BN; col += 16) {
                uint32_t v[16];
                __syncwarp();
                tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + col, v);
                tmem_ld_wait();
                if (row_ok) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int nl = col + i;
                        const int n = n0 + nl;
                        if (n < N) {
                            const int32_t a = static_cast<int32_t>(v[i]);
                            float y = __fmul_rn(__fmul_rn(static_cast<float>(a), sxm), s_sw[nl]);
                            y += s_bias[nl];
                            float l = 0.f;
#pragma unroll
                            for (int j = 0; j < RMAX; ++j) {
                                if (j < ep.r) {
                                    const float b = kStageB ? s_lb[j * BN + nl]
                                                            : __ldg(ep.B + static_cast<size_t>(j) * N + n);
                                    l = fmaf(xa[j], b, l);
                                }
                            }
                            store_out<OutT>(yrow + n, y + l);
                            if (arow) arow[n] = a;
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, BN);
    }
}

template <int BN, int STAGES, typename OutT, int RMAX>
cudaError_t launch_cfg(const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K,
                       const FwdEpilogue& ep, int* status, cudaStream_t s) {
    using L = K2Layout<BN, STAGES>;
    auto kern = k2_gemm_i8_lora_kernel<BN, STAGES, OutT, RMAX>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), L::kTotal);
    if (e != cudaSuccess) return e;
    dim3 grid((N + BN - 1) / BN, (M + kBM - 1) / kBM);
    kern<<<grid, kThreads, L::kTotal, s>>>(ta, tb, M, N, K, ep, status);
    return cudaGetLastError();
}

template <typename OutT, int RMAX>
cudaError_t launch_bn(int bn, const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K,
                      const FwdEpilogue& ep, int* status, cudaStream_t s) {
    if (bn == 256) return launch_cfg<256, 4, OutT, RMAX>(ta, tb, M, N, K, ep, status, s);
    if (bn == 128) return launch_cfg<128, 6, OutT, RMAX>(ta, tb, M, N, K, ep, status, s);
    return launch_cfg<64, 8, OutT, RMAX>(ta, tb, M, N, K, ep, status, s);
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
    // Tile width: the widest BN that still gives about one tile per SM.
    const int mt = (M + kBM - 1) / kBM;
    int bn = 256;
    while (bn > 64 && mt * ((N + bn - 1) / bn) < 148) bn /= 2;
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
