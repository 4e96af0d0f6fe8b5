// k3_dx.cu -- input gradient of the int8-LoRA Dense layer:
//
//   dX[m,k] = sum_n dY[m,n] * bf16(Wq[n,k] * sw[n]) + c * sum_j G[m,j] A[k,j]
//
// The frozen int8 kernel is de-quantized tile by tile in shared memory right
// before the tensor-core product ("How to fine-tune the 4-bit model?"
// thread: decompress the quantized weights in place, then feed the matrix
// unit; the de-quantization cost is paid per batch, not per input).  The
// input quantizer is passed straight through, so only the de-quantized
// kernel and the LoRA factors enter dX.
//
// tcgen05 path (bf16 activations, N a multiple of 8), one 128 x BN tile of dX
// per CTA, 10 warps:
//   warp 0      TMA producer: dY tile [128 x 64 bf16] (128B swizzle, K-major)
//               and the int8 kernel tile Wq[n0:n0+64, k0:k0+BN] (row-major)
//   warp 1      TMEM allocation; tcgen05.mma.kind::f16 (bf16 in, fp32 accum),
//               M=128, N=BN, K=16 per instruction, from one thread
//   warps 2..9  de-quantize each int8 stage into a bf16 tile laid out as the
//               MN-major 128B-swizzled B operand, then run the epilogue
// SIMT path: fp32 activations, or rows of dY that the Tensor Memory
// Accelerator cannot describe (N*2 bytes not a multiple of 16).
#include "internal.h"
#include "ptx.cuh"

namespace qlora {

namespace {

constexpr int kBM = 128;
constexpr int kBKn = 64;  // contraction (n) per stage: one 128-byte row of bf16
constexpr int kDqWarps = 8;
constexpr int kThreads = 64 + 32 * kDqWarps;

template <int BN, int STAGES>
struct K3Layout {
    static constexpr int kABytes = kBM * kBKn * 2;     // dY tile, bf16
    static constexpr int kQBytes = kBKn * BN;          // int8 kernel tile
    static constexpr int kWBytes = kBKn * BN * 2;      // de-quantized bf16 tile
    static constexpr int kStageBytes = kABytes + kQBytes + kWBytes;
    static constexpr int kBarOff = STAGES * kStageBytes;
    static constexpr int kLoraOff = kBarOff + 256;     // A tile [BN][16]
    static constexpr int kTotal = kLoraOff + BN * 16 * 4 + 1024;
};

// byte offset of the 16-byte chunk holding bf16 elements (mn .. mn+7, kr) in
// an MN-major, 128B-swizzled operand tile with 8-row K groups 1024 B apart and
// 64-element MN blocks `lbo` bytes apart.
__device__ __forceinline__ uint32_t mn_sw128_offset(int mn, int kr, uint32_t lbo) {
    const int mb = mn >> 6;
    const int chunk = (mn & 63) >> 3;
    const int kg = kr >> 3;
    const int row = kr & 7;
    return mb * lbo + kg * 1024 + row * 128 + ((chunk ^ row) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <int BN, int STAGES, int RMAX>
__global__ void __launch_bounds__(kThreads, 1)
    k3_dx_dequant_kernel(const __grid_constant__ CUtensorMap tmDY,
                         const __grid_constant__ CUtensorMap tmQ, const float* __restrict__ sw,
                         int M, int N, int K, DxEpilogue ep, int* status) {
    using L = K3Layout<BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* wready = full + STAGES;
    uint64_t* empty = wready + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 1);
    float* s_a = reinterpret_cast<float*>(smem + L::kLoraOff);
    constexpr bool kStageA = RMAX <= 16;
    constexpr uint32_t kLbo = (kBKn / 8) * 1024;  // MN-block stride of the bf16 tile

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int m0 = blockIdx.y * kBM;
    const int k0 = blockIdx.x * BN;
    const int nkb = (N + kBKn - 1) / kBKn;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&wready[s], kDqWarps);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, BN);
        tmem_relinquish();
    }
    if constexpr (kStageA) {
        for (int i = threadIdx.x; i < BN * RMAX; i += kThreads) {
            const int kk = i / RMAX, j = i % RMAX;
            const int k = k0 + kk;
            s_a[i] = (k < K && j < ep.r) ? ep.A[static_cast<size_t>(k) * ep.r + j] : 0.f;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tmDY);
            tma_prefetch_desc(&tmQ);
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % STAGES;
                const int it = kb / STAGES;
                if (kb >= STAGES && !mbar_wait(&empty[s], (it - 1) & 1, status)) break;
                uint8_t* sa = smem + s * L::kStageBytes;
                uint8_t* sq = sa + L::kABytes;
                mbar_arrive_expect_tx(&full[s], L::kABytes + L::kQBytes);
                tma_load_2d(sa, &tmDY, &full[s], kb * kBKn, m0);
                tma_load_2d(sq, &tmQ, &full[s], k0, kb * kBKn);
            }
        }
        __syncwarp();  // reconverge the warp before the teardown barrier
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(kBM, BN, false, true);
            bool ok = true;
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % STAGES;
                const int it = kb / STAGES;
                if (!mbar_wait(&full[s], it & 1, status) || !mbar_wait(&wready[s], it & 1, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_base = smem_u32(smem + s * L::kStageBytes);
                const uint32_t w_base = a_base + L::kABytes + L::kQBytes;
#pragma unroll
                for (int kk = 0; kk < kBKn / 16; ++kk) {
                    const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024, kLayoutSw128);
                    const uint64_t bd = smem_desc(w_base + kk * 2048, kLbo, 1024, kLayoutSw128);
                    mma_bf16(tmem, ad, bd, idesc, (kb | kk) != 0);
                }
                mma_commit(&empty[s]);
            }
            if (ok) mma_commit(tfull);
        }
        __syncwarp();  // reconverge the warp before the teardown barrier
    } else {
        const int dq = threadIdx.x - 64;  // 0 .. 255
        // ---- de-quantize every stage into the MN-major swizzled bf16 tile ----
        constexpr int kChunksPerRow = BN / 16;
        constexpr int kChunks = kBKn * kChunksPerRow;
        bool ok = true;
        for (int kb = 0; kb < nkb && ok; ++kb) {
            const int s = kb % STAGES;
            const int it = kb / STAGES;
            ok = __all_sync(0xffffffffu, mbar_wait(&full[s], it & 1, status));
            if (!ok) break;
            const uint8_t* sq = smem + s * L::kStageBytes + L::kABytes;
            uint8_t* sw_tile = smem + s * L::kStageBytes + L::kABytes + L::kQBytes;
#pragma unroll
            for (int c = dq; c < kChunks; c += 32 * kDqWarps) {
                const int nr = c / kChunksPerRow;   // contraction row within the stage
                const int kc = c % kChunksPerRow;   // 16 output columns
                const int n = kb * kBKn + nr;
                const float scale = n < N ? __ldg(sw + n) : 0.f;
                const uint4 raw = *reinterpret_cast<const uint4*>(sq + nr * BN + kc * 16);
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
                uint32_t o[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int32_t b = static_cast<int32_t>(w4[i]);
                    const float f0 = __fmul_rn(static_cast<float>((b << 24) >> 24), scale);
                    const float f1 = __fmul_rn(static_cast<float>((b << 16) >> 24), scale);
                    const float f2 = __fmul_rn(static_cast<float>((b << 8) >> 24), scale);
                    const float f3 = __fmul_rn(static_cast<float>(b >> 24), scale);
                    o[2 * i] = pack_bf16x2(f0, f1);
                    o[2 * i + 1] = pack_bf16x2(f2, f3);
                }
                const int mn = kc * 16;
                *reinterpret_cast<uint4*>(sw_tile + mn_sw128_offset(mn, nr, kLbo)) =
                    make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4*>(sw_tile + mn_sw128_offset(mn + 8, nr, kLbo)) =
                    make_uint4(o[4], o[5], o[6], o[7]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&wready[s]);
        }
        // ---- epilogue ----
        const int q = warp & 3;
        const int half = (warp - 2) / 4;
        const int row = m0 + q * 32 + lane;
        const bool row_ok = row < M;
        float g[RMAX];
#pragma unroll
        for (int j = 0; j < RMAX; ++j)
            g[j] = (row_ok && j < ep.r) ? ep.G[static_cast<size_t>(row) * ep.r + j] * ep.c : 0.f;
        ok = __all_sync(0xffffffffu, ok && mbar_wait(tfull, 0, status));
        tc_fence_after();
        if (ok) {
            __nv_bfloat16* drow =
                static_cast<__nv_bfloat16*>(ep.dX) + static_cast<size_t>(row_ok ? row : 0) * K;
#pragma unroll 1
            for (int col = half * (BN / 2); col < (half + 1) * (BN / 2); col += 16) {
                uint32_t v[16];
                __syncwarp();
                tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + col, v);
                tmem_ld_wait();
                if (row_ok) {
                    float outv[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int kl = col + i;
                        const int k = k0 + kl;
                        float l = 0.f;
#pragma unroll
                        for (int j = 0; j < RMAX; ++j) {
                            if (j < ep.r) {
                                const float a = kStageA ? s_a[kl * RMAX + j]
                                                        : (k < K ? __ldg(ep.A + static_cast<size_t>(k) * ep.r + j) : 0.f);
                                l = fmaf(g[j], a, l);
                            }
                        }
                        outv[i] = __uint_as_float(v[i]) + l;
                    }
                    const int kbase = k0 + col;
                    if (kbase + 16 <= K) {
                        uint4 p0 = make_uint4(pack_bf16x2(outv[0], outv[1]), pack_bf16x2(outv[2], outv[3]),
                                              pack_bf16x2(outv[4], outv[5]), pack_bf16x2(outv[6], outv[7]));
                        uint4 p1 = make_uint4(pack_bf16x2(outv[8], outv[9]), pack_bf16x2(outv[10], outv[11]),
                                              pack_bf16x2(outv[12], outv[13]), pack_bf16x2(outv[14], outv[15]));
                        *reinterpret_cast<uint4*>(drow + kbase) = p0;
                        *reinterpret_cast<uint4*>(drow + kbase + 8) = p1;
                    } else {
                        for (int i = 0; i < 16; ++i)
                            if (kbase + i < K) drow[kbase + i] = __float2bfloat16_rn(outv[i]);
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

template <int BN, int STAGES, int RMAX>
cudaError_t launch_tc(const CUtensorMap& tdy, const CUtensorMap& tq, const float* sw, int M, int N,
                      int K, const DxEpilogue& ep, int* status, cudaStream_t s) {
    using L = K3Layout<BN, STAGES>;
    auto kern = k3_dx_dequant_kernel<BN, STAGES, RMAX>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), L::kTotal);
    if (e != cudaSuccess) return e;
    dim3 grid((K + BN - 1) / BN, (M + kBM - 1) / kBM);
    kern<<<grid, kThreads, L::kTotal, s>>>(tdy, tq, sw, M, N, K, ep, status);
    return cudaGetLastError();
}

template <int RMAX>
cudaError_t launch_tc_bn(int bn, const CUtensorMap& tdy, const CUtensorMap& tq, const float* sw,
                         int M, int N, int K, const DxEpilogue& ep, int* status, cudaStream_t s) {
    if (bn == 256) return launch_tc<256, 3, RMAX>(tdy, tq, sw, M, N, K, ep, status, s);
    return launch_tc<128, 5, RMAX>(tdy, tq, sw, M, N, K, ep, status, s);
}

// ---------------------------------------------------------------- SIMT path
// 64 x 64 tile of dX per CTA, 256 threads (4 x 4 outputs each), n in steps of
// 16 through shared memory; the kernel tile is de-quantized to fp32 on load.
constexpr int kSB = 64;
constexpr int kSN = 16;

template <typename T>
__global__ void __launch_bounds__(256) k3_dx_simt_kernel(const T* __restrict__ dY,
                                                         const int8_t* __restrict__ Wq,
                                                         const float* __restrict__ sw, int M,
                                                         int N, int K, DxEpilogue ep) {
    __shared__ float sD[kSN][kSB + 1];  // [n][m]
    __shared__ float sW[kSN][kSB + 1];  // [n][k]
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int m0 = blockIdx.y * kSB, k0 = blockIdx.x * kSB;
    float acc[4][4] = {};
    for (int n0 = 0; n0 < N; n0 += kSN) {
        for (int i = threadIdx.x; i < kSN * kSB; i += 256) {
            const int mm = i / kSN, nn = i % kSN;  // consecutive threads: consecutive n of a row
            const int m = m0 + mm, n = n0 + nn;
            sD[nn][mm] = (m < M && n < N) ? ActIO<T>::to_f(dY[static_cast<size_t>(m) * N + n]) : 0.f;
        }
        for (int i = threadIdx.x; i < kSN * kSB; i += 256) {
            const int nn = i / kSB, kk = i % kSB;
            const int n = n0 + nn, k = k0 + kk;
            sW[nn][kk] = (n < N && k < K)
                             ? __fmul_rn(static_cast<float>(Wq[static_cast<size_t>(n) * K + k]), __ldg(sw + n))
                             : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int nn = 0; nn < kSN; ++nn) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = sD[nn][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = sW[nn][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    T* dX = static_cast<T*>(ep.dX);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty + 16 * i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = k0 + tx + 16 * j;
            if (k >= K) continue;
            float l = 0.f;
            for (int jj = 0; jj < ep.r; ++jj)
                l = fmaf(ep.G[static_cast<size_t>(m) * ep.r + jj], ep.A[static_cast<size_t>(k) * ep.r + jj], l);
            dX[static_cast<size_t>(m) * K + k] = ActIO<T>::from_f(acc[i][j] + ep.c * l);
        }
    }
}

}  // namespace

cudaError_t launch_gemm_dx(Act act, const void* dY, const int8_t* Wq, const float* sw, int M,
                           int N, int K, const DxEpilogue& ep, int* status, cudaStream_t s) {
    const bool tc = act == kBF16 && (N % 8) == 0;
    if (!tc) {
        dim3 grid((K + kSB - 1) / kSB, (M + kSB - 1) / kSB);
        if (act == kBF16)
            k3_dx_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
                static_cast<const __nv_bfloat16*>(dY), Wq, sw, M, N, K, ep);
        else
            k3_dx_simt_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(dY), Wq, sw, M, N,
                                                          K, ep);
        return cudaGetLastError();
    }
    const int mt = (M + kBM - 1) / kBM;
    const int bn = (mt * ((K + 255) / 256) >= 148) ? 256 : 128;
    CUtensorMap tdy, tq;
    if (!make_tmap_2d(&tdy, dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N,
                      static_cast<uint64_t>(N) * 2, kBM, kBKn, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_tmap_2d(&tq, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, K, kBKn, bn,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (ep.r <= 4) return launch_tc_bn<4>(bn, tdy, tq, sw, M, N, K, ep, status, s);
    if (ep.r <= 8) return launch_tc_bn<8>(bn, tdy, tq, sw, M, N, K, ep, status, s);
    if (ep.r <= 16) return launch_tc_bn<16>(bn, tdy, tq, sw, M, N, K, ep, status, s);
    return launch_tc_bn<64>(bn, tdy, tq, sw, M, N, K, ep, status, s);
}

}  // namespace qlora
