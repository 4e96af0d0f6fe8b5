// fp8.cu -- the float8 training recipe ("Introduce float8 training", Keras
// PR 19488: quantization mode "float8", per-tensor scales and amax
// histories updated every step, float8 matmuls on float8 tensor cores).
//
// Readings (the page prints no formula; stated once here, restated in the
// C header): inputs and kernel in E4M3, the output gradient in E5M2; a
// tensor T is quantized with the scale stored by the previous step,
//   q = fp8(satfinite(fl32(T / s)))        round to nearest, ties to even,
// and the step then stores s' = fl32(h / fp8_max) (h the largest entry of
// the amax history before this step; s' = s when h is 0 or not finite) and
// the history [amax(|T|), H[0], .., H[L-2]].  The GEMMs multiply the codes
// on tcgen05.mma.kind::f8f6f4 (fp32 accumulate) and scale the result by the
// product of the two operands' scales.
//
// Kernels:
//   fp8_quantize_kernel  32 x 32 tiles of T: codes row-major and, through
//                        shared memory, transposed (the K-major operand of
//                        the backward GEMMs); |T|'s maximum by atomicMax on
//                        the float bits (non-negative floats order as
//                        unsigned integers)
//   fp8_state_kernel     one block: the new scale and the rolled history
//   fp8_gemm_kernel      C = (A B^T) sa sb (+ bias): one 128 x 256 (or 128 x
//                        128) tile per CTA, both operands K-major fp8 by TMA
//                        (128-byte swizzle, 128 k per stage), 4 MMAs of
//                        K = 32 per stage into a TMEM accumulator, four
//                        epilogue warps
#include "internal.h"
#include "ptx.cuh"
#include "tile_epilogue.cuh"

#include <cuda_fp8.h>

namespace qlora {

namespace {

__device__ __forceinline__ uint8_t to_fp8(float v, int fmt) {
    return fmt == kFp8E4M3 ? static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3))
                           : static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E5M2));
}

constexpr int kQT = 32;

template <typename T>
__global__ void __launch_bounds__(256) fp8_quantize_kernel(const T* __restrict__ src, int R, int Cc,
                                                          const float* __restrict__ scale, int fmt,
                                                          uint8_t* __restrict__ q, uint8_t* __restrict__ qt,
                                                          unsigned int* __restrict__ amax_bits) {
    __shared__ uint8_t tile[kQT][kQT + 4];
    pdl_trigger();
    pdl_wait();
    const float s = __ldg(scale);
    const int r0 = blockIdx.y * kQT, c0 = blockIdx.x * kQT;
    const int tx = threadIdx.x % kQT, ty = threadIdx.x / kQT;  // 32 x 8
    float mx = 0.f;
    for (int rr = ty; rr < kQT; rr += 8) {
        const int r = r0 + rr, c = c0 + tx;
        uint8_t code = 0;
        if (r < R && c < Cc) {
            const float v = ActIO<T>::to_f(src[static_cast<size_t>(r) * Cc + c]);
            mx = fmaxf(mx, fabsf(v));
            code = to_fp8(__fdiv_rn(v, s), fmt);
            q[static_cast<size_t>(r) * Cc + c] = code;
        }
        tile[rr][tx] = code;
    }
    // block maximum, then one atomic per block
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    __shared__ float wmax[8];
    if (tx == 0) wmax[ty] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = wmax[0];
        for (int i = 1; i < 8; ++i) m = fmaxf(m, wmax[i]);
        atomicMax(amax_bits, __float_as_uint(m));
    }
    if (qt) {
        for (int cc = ty; cc < kQT; cc += 8) {
            const int c = c0 + cc, r = r0 + tx;
            if (c < Cc && r < R) qt[static_cast<size_t>(c) * R + r] = tile[tx][cc];
        }
    }
}

// new scale from the history before this step, then the rolled history
__global__ void __launch_bounds__(1024) fp8_state_kernel(const unsigned int* __restrict__ amax_bits,
                                                        const float* __restrict__ scale_in,
                                                        float* __restrict__ scale_out,
                                                        float* __restrict__ hist, int L, float fmax) {
    pdl_trigger();
    pdl_wait();
    __shared__ float red[32];
    float m = -INFINITY;
    bool finite = true;
    for (int i = threadIdx.x; i < L; i += blockDim.x) {
        const float h = hist[i];
        finite = finite && isfinite(h);
        m = fmaxf(m, h);
    }
    finite = __syncthreads_and(finite);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float h = red[0];
        for (int i = 1; i < static_cast<int>((blockDim.x + 31) / 32); ++i) h = fmaxf(h, red[i]);
        const float s = __ldg(scale_in);
        *scale_out = (finite && h > 0.f) ? __fdiv_rn(h, fmax) : s;
    }
    // shift by one, newest first, one chunk of blockDim entries at a time
    // from the back: a chunk reads its own entries and the last entry of the
    // chunk before it, neither written yet
    const int nchunks = (L + static_cast<int>(blockDim.x) - 1) / static_cast<int>(blockDim.x);
    for (int ch = nchunks - 1; ch >= 0; --ch) {
        const int i = ch * static_cast<int>(blockDim.x) + static_cast<int>(threadIdx.x);
        const float prev = (i >= 1 && i < L) ? hist[i - 1] : 0.f;
        __syncthreads();
        if (i >= 1 && i < L) hist[i] = prev;
        __syncthreads();
    }
    if (threadIdx.x == 0) hist[0] = __uint_as_float(*amax_bits);
}

}  // namespace

namespace {

constexpr int kGM = 128, kGK = 128;  // tile rows, k bytes per stage
constexpr int kGEpi = 4;
constexpr int kGThreads = 32 * (2 + kGEpi);
// BN = 256 columns per tile where the output is wide enough (an MMA of
// N = 256 keeps the tensor pipe busy for about as long as one takes to
// issue), else 128; as many stages as fit 192 KB.
template <int BN>
struct GCfg {
    static constexpr uint32_t kStage = (kGM + BN) * kGK;
    static constexpr int kStages = (192 * 1024) / kStage > 8 ? 8 : (192 * 1024) / kStage;
};

// kind::f8f6f4 instruction descriptor: fp32 D; A and B formats (E4M3 0,
// E5M2 1) in bits [7,10) and [10,13); both K-major; N >> 3, M >> 4.
__host__ __device__ constexpr uint32_t idesc_f8(int m, int n, int afmt, int bfmt) {
    return (1u << 4) | (static_cast<uint32_t>(afmt) << 7) | (static_cast<uint32_t>(bfmt) << 10) |
           (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <typename OutT, int BN>
__global__ void __launch_bounds__(kGThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M,
                    int N, int K, uint32_t idesc, const float* __restrict__ sa, const float* __restrict__ sb,
                    const float* __restrict__ bias, OutT* __restrict__ C, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    constexpr int kGStages = GCfg<BN>::kStages;
    constexpr uint32_t kGStage = GCfg<BN>::kStage;
    constexpr int kGN = BN;
    constexpr uint32_t kStgOff = kGStages * kGStage;
    constexpr uint32_t kBarOff = kStgOff + kGEpi * 32 * stage_pitch<OutT>();
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);
    uint64_t* empty = full + kGStages;
    uint64_t* accf = empty + kGStages;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(accf + 1);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int n0 = blockIdx.x * kGN, m0 = blockIdx.y * kGM;
    const int nkb = (K + kGK - 1) / kGK;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tslot, BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    pdl_trigger();
    pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            for (int i = 0; i < nkb; ++i) {
                const int s = i % kGStages;
                if (i >= kGStages && !mbar_wait(&empty[s], ((i / kGStages) - 1) & 1, status)) break;
                uint8_t* st = smem + s * kGStage;
                mbar_arrive_expect_tx(&full[s], kGStage);
                tma_load_2d(st, &tmA, &full[s], i * kGK, m0);
                tma_load_2d(st + kGM * kGK, &tmB, &full[s], i * kGK, n0);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            for (int i = 0; i < nkb; ++i) {
                const int s = i % kGStages;
                if (!mbar_wait(&full[s], (i / kGStages) & 1, status)) break;
                tc_fence_after();
                const uint32_t ab = smem_u32(smem + s * kGStage);
                const uint32_t bb = ab + kGM * kGK;
#pragma unroll
                for (int kk = 0; kk < kGK / 32; ++kk) {
                    const uint64_t ad = smem_desc(ab + kk * 32, 16, 1024, kLayoutSw128);
                    const uint64_t bd = smem_desc(bb + kk * 32, 16, 1024, kLayoutSw128);
                    mma_f8(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&empty[s]);
            }
            mma_commit(accf);
        }
        __syncwarp();
    } else {
        const int q = warp & 3;  // the TMEM lane quarter this warp may access
        const bool ok = __all_sync(0xffffffffu, mbar_wait(accf, 0, status));
        tc_fence_after();
        const float sab = __fmul_rn(__ldg(sa), __ldg(sb));
        uint8_t* stg = smem + kStgOff + (warp - 2) * 32 * stage_pitch<OutT>();
        const int row0 = m0 + q * 32;
        const bool vec = ((static_cast<size_t>(N) * sizeof(OutT)) % 16) == 0;
        if (ok && nkb > 0) {
            for (int col = 0; col < kGN; col += kEpiCols) {
                uint32_t v[kEpiCols];
                tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + col, v);
                tmem_ld_wait();
                float y[kEpiCols];
#pragma unroll
                for (int e = 0; e < kEpiCols; ++e) {
                    const int n = n0 + col + e;
                    const float b = (bias && n < N) ? __ldg(bias + n) : 0.f;
                    y[e] = fmaf(__uint_as_float(v[e]), sab, b);
                }
                store_block<OutT>(stg, y, lane, C, static_cast<size_t>(N), row0, M, n0 + col, N, vec);
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

}  // namespace

cudaError_t launch_fp8_quantize(Act act, const void* T, int R, int Cc, const float* scale_in, float* scale_out,
                                float* hist, int L, int fmt, uint8_t* q, uint8_t* qt, unsigned int* amax_word,
                                cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(amax_word, 0, sizeof(unsigned int), s);
    if (e != cudaSuccess) return e;
    const dim3 grid((Cc + kQT - 1) / kQT, (R + kQT - 1) / kQT);
    e = act == kBF16
            ? launch_k(fp8_quantize_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, 1,
                       static_cast<const __nv_bfloat16*>(T), R, Cc, scale_in, fmt, q, qt, amax_word)
            : launch_k(fp8_quantize_kernel<float>, grid, dim3(256), 0, s, 1, static_cast<const float*>(T), R,
                       Cc, scale_in, fmt, q, qt, amax_word);
    if (e != cudaSuccess) return e;
    const float fmax = fmt == kFp8E4M3 ? 448.0f : 57344.0f;
    return launch_k(fp8_state_kernel, dim3(1), dim3(1024), 0, s, 1, static_cast<const unsigned int*>(amax_word),
                    scale_in, scale_out, hist, L, fmax);
}

cudaError_t launch_fp8_gemm(const uint8_t* A, int afmt, const uint8_t* B, int bfmt, int M, int N, int K,
                            const float* sa, const float* sb, const float* bias, void* C, Act out, int* status,
                            cudaStream_t s) {
    CUtensorMap ta, tb;
    if (!make_tmap_2d(&ta, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K, K, kGM, kGK, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tb, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, K, 128, kGK, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int bn = N >= 256 ? 256 : 128;
    CUtensorMap tb2;
    if (!make_tmap_2d(&tb2, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, K, bn, kGK, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    (void)tb;
    const uint32_t id = idesc_f8(kGM, bn, afmt, bfmt);
    const dim3 grid((N + bn - 1) / bn, (M + kGM - 1) / kGM);
    auto run = [&](auto kern, size_t stage_bytes_total, size_t pitch) -> cudaError_t {
        const size_t smem = stage_bytes_total + kGEpi * 32 * pitch + 256 + 1024;
        cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        return launch_k(kern, grid, dim3(kGThreads), smem, s, 1, ta, tb2, M, N, K, id, sa, sb, bias, C, status);
    };
    constexpr size_t r128 = static_cast<size_t>(GCfg<128>::kStages) * GCfg<128>::kStage;
    constexpr size_t r256 = static_cast<size_t>(GCfg<256>::kStages) * GCfg<256>::kStage;
    if (out == kBF16)
        return bn == 256 ? run(fp8_gemm_kernel<__nv_bfloat16, 256>, r256, stage_pitch<__nv_bfloat16>())
                         : run(fp8_gemm_kernel<__nv_bfloat16, 128>, r128, stage_pitch<__nv_bfloat16>());
    return bn == 256 ? run(fp8_gemm_kernel<float, 256>, r256, stage_pitch<float>())
                     : run(fp8_gemm_kernel<float, 128>, r128, stage_pitch<float>());
}

}  // namespace qlora
