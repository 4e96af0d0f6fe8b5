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
    const int r0 = blockIdx.x * kQT, c0 = blockIdx.y * kQT;
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

// The same quantizer for aligned layouts (T 16-byte aligned, cols % 8 == 0,
// q 8-byte aligned; qt 16-byte aligned with rows % 16 == 0): one 128 x 128
// tile per block of 256 threads.  Each thread loads eight 8-value chunks
// (16-byte loads, all in flight before the first is used), converts two
// values per cvt and stores 8 codes per 8-byte store; the codes also go to
// a 16 KB shared tile (32 words a row, word w of row r at w ^ 4 ((r / 16) %
// 8), so that both the 8-byte stores and the column reads below are free of
// bank conflicts).  For qt each thread then reads a 16-row x 4-column block,
// transposes it four 4 x 4 byte blocks at a time with byte permutes and
// writes four 16-byte runs of qt rows; eight threads cover 128 contiguous
// bytes of one qt row.
constexpr int kFR = 128, kFC = 128, kFThreads = 256;
constexpr int kFChunks = kFR * kFC / 8 / kFThreads;  // 8 chunks of 8 values per thread

__device__ __forceinline__ void load8(const __nv_bfloat16* p, uint32_t (&raw)[8]) {
    const uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
    raw[0] = r.x;
    raw[1] = r.y;
    raw[2] = r.z;
    raw[3] = r.w;
}
__device__ __forceinline__ void load8(const float* p, uint32_t (&raw)[8]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    raw[0] = a.x;
    raw[1] = a.y;
    raw[2] = a.z;
    raw[3] = a.w;
    raw[4] = b.x;
    raw[5] = b.y;
    raw[6] = b.z;
    raw[7] = b.w;
}
__device__ __forceinline__ float val8(const uint32_t (&raw)[8], int i, const __nv_bfloat16*) {
    return __uint_as_float((i & 1) ? (raw[i >> 1] & 0xffff0000u) : (raw[i >> 1] << 16));
}
__device__ __forceinline__ float val8(const uint32_t (&raw)[8], int i, const float*) {
    return __uint_as_float(raw[i]);
}

template <int FMT>
__device__ __forceinline__ uint32_t cvt2(float lo, float hi) {
    const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE,
                                                            FMT == kFp8E4M3 ? __NV_E4M3 : __NV_E5M2);
    return static_cast<uint32_t>(c);
}

// rows (w0..w3) x 4 byte columns -> 4 columns (c0..c3) x 4 rows
__device__ __forceinline__ void transpose4x4(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, uint32_t& c0,
                                             uint32_t& c1, uint32_t& c2, uint32_t& c3) {
    const uint32_t t0 = __byte_perm(w0, w1, 0x5140);  // w0.b0 w1.b0 w0.b1 w1.b1
    const uint32_t t1 = __byte_perm(w0, w1, 0x7362);  // w0.b2 w1.b2 w0.b3 w1.b3
    const uint32_t t2 = __byte_perm(w2, w3, 0x5140);
    const uint32_t t3 = __byte_perm(w2, w3, 0x7362);
    c0 = __byte_perm(t0, t2, 0x5410);
    c1 = __byte_perm(t0, t2, 0x7632);
    c2 = __byte_perm(t1, t3, 0x5410);
    c3 = __byte_perm(t1, t3, 0x7632);
}

// Column sums (CS): each thread adds its 8 columns over its 8 rows, the 16
// threads of a column chunk are added in a fixed order through shared
// memory, and the tile's sums go to part[row tile][col]; a second kernel
// (fp8_colsum_kernel) adds each column's partials over the row tiles in a
// fixed order.  (Doing that last step in the last block of each column strip needs
// a device-scope fence in every block, which measured slower than the extra
// launch.)
template <typename T, int FMT, bool CS>
__global__ void __launch_bounds__(kFThreads) fp8_quantize_tiled_kernel(const T* __restrict__ src, int R, int Cc,
                                                                      const float* __restrict__ scale,
                                                                      uint8_t* __restrict__ q,
                                                                      uint8_t* __restrict__ qt,
                                                                      unsigned int* __restrict__ amax_bits,
                                                                      float* __restrict__ part) {
    __shared__ __align__(16) uint32_t tile[kFR * kFC / 4];
    __shared__ __align__(16) float csm[CS ? 16 * kFC : 1];
    __shared__ float wmax[kFThreads / 32];
    pdl_trigger();
    pdl_wait();
    const int t = threadIdx.x;
    const int r0 = blockIdx.x * kFR, c0 = blockIdx.y * kFC;
    const int j = t % 16;  // this thread's 8-column chunk in every row it handles
    const int gc = c0 + 8 * j;
    uint32_t raw[kFChunks][8];
#pragma unroll
    for (int u = 0; u < kFChunks; ++u) {
        const int gr = r0 + t / 16 + 16 * u;
        if (gr < R && gc < Cc) load8(src + static_cast<size_t>(gr) * Cc + gc, raw[u]);
        else
#pragma unroll
            for (int i = 0; i < 8; ++i) raw[u][i] = 0u;
    }
    const float s = __ldg(scale);
    float mx = 0.f;
    float cs[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) cs[i] = 0.f;
#pragma unroll
    for (int u = 0; u < kFChunks; ++u) {
        const int row = t / 16 + 16 * u;
        const int gr = r0 + row;
        float x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float v = val8(raw[u], i, src);
            mx = fmaxf(mx, fabsf(v));
            if constexpr (CS) cs[i] += v;
            x[i] = __fdiv_rn(v, s);
        }
        const uint32_t lo = cvt2<FMT>(x[0], x[1]) | (cvt2<FMT>(x[2], x[3]) << 16);
        const uint32_t hi = cvt2<FMT>(x[4], x[5]) | (cvt2<FMT>(x[6], x[7]) << 16);
        if (gr < R && gc < Cc)
            *reinterpret_cast<uint2*>(q + static_cast<size_t>(gr) * Cc + gc) = make_uint2(lo, hi);
        const int w = (2 * j) ^ (((row >> 4) & 7) << 2);
        *reinterpret_cast<uint2*>(&tile[row * 32 + w]) = make_uint2(lo, hi);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (t % 32 == 0) wmax[t / 32] = mx;
    if constexpr (CS) {
        float4* d = reinterpret_cast<float4*>(&csm[(t / 16) * kFC + 8 * j]);
        d[0] = make_float4(cs[0], cs[1], cs[2], cs[3]);
        d[1] = make_float4(cs[4], cs[5], cs[6], cs[7]);
    }
    __syncthreads();
    if (t == 0) {
        float m = wmax[0];
#pragma unroll
        for (int i = 1; i < kFThreads / 32; ++i) m = fmaxf(m, wmax[i]);
        atomicMax(amax_bits, __float_as_uint(m));
    }
    if constexpr (CS) {
        if (t < kFC) {
            float p = 0.f;
#pragma unroll
            for (int k = 0; k < 16; ++k) p += csm[k * kFC + t];
            if (c0 + t < Cc) part[static_cast<size_t>(blockIdx.x) * Cc + c0 + t] = p;
        }
    }
    if (qt) {
        const int seg = t % 8, c4 = t / 8;
        const int gr = r0 + 16 * seg;
        if (gr < R) {
            uint32_t col[4][4];  // [column of the quad][group of 4 rows]
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) w[i] = tile[(16 * seg + 4 * g + i) * 32 + (c4 ^ (seg << 2))];
                transpose4x4(w[0], w[1], w[2], w[3], col[0][g], col[1][g], col[2][g], col[3][g]);
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int c = c0 + 4 * c4 + jj;
                if (c < Cc)
                    *reinterpret_cast<uint4*>(qt + static_cast<size_t>(c) * R + gr) =
                        make_uint4(col[jj][0], col[jj][1], col[jj][2], col[jj][3]);
            }
        }
    }
}

// colsum[c] = sum over row tiles of part[t][c] in a fixed order: a block
// takes 32 columns; its eight warps each add one eighth of the row tiles
// (ascending, eight loads in flight), then one warp adds the eight sums in
// warp order.
constexpr int kCsCols = 32, kCsWarps = 8;
__global__ void __launch_bounds__(32 * kCsWarps) fp8_colsum_kernel(const float* __restrict__ part, int nrt, int Cc,
                                                                  float* __restrict__ colsum) {
    __shared__ float sums[kCsWarps][kCsCols];
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x % 32, w = threadIdx.x / 32;
    const int c = blockIdx.x * kCsCols + lane;
    const int per = (nrt + kCsWarps - 1) / kCsWarps;
    const int t0 = w * per, t1 = min(nrt, t0 + per);
    float v = 0.f;
    if (c < Cc) {
        int t = t0;
        for (; t + 8 <= t1; t += 8) {
            float x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) x[u] = __ldg(part + static_cast<size_t>(t + u) * Cc + c);
#pragma unroll
            for (int u = 0; u < 8; ++u) v += x[u];
        }
        for (; t < t1; ++t) v += __ldg(part + static_cast<size_t>(t) * Cc + c);
    }
    sums[w][lane] = v;
    __syncthreads();
    if (w == 0 && c < Cc) {
        float a = sums[0][lane];
#pragma unroll
        for (int k = 1; k < kCsWarps; ++k) a += sums[k][lane];
        colsum[c] = a;
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

// ---------------------------------------------------------------------------
// The same product on CTA pairs, for outputs of at least one 256 x 256 tile
// per pair of SMs: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2.kind::f8f6f4 (M = 256, N = 256, K = 32); CTA r
// loads A rows [128 r, +128) and B rows [128 r, +128) of the tile, 128 k per
// stage (TMA, K-major, 128-byte swizzle) and holds its 128 rows x 256 columns
// of the fp32 accumulator in TMEM.  Each CTA then streams half as many bytes
// per MMA as in the one-CTA kernel.  Persistent: pair p takes tiles p,
// p + pairs, ...; the accumulator is double-buffered (512 TMEM columns) so
// the epilogue of one tile overlaps the main loop of the next.
// Warps: 0 TMA producer; 1 TMEM owner and, in CTA 0, the MMA issuer; 2..5
// epilogue.  full[s] (CTA 0) completes when the four boxes of stage s have
// landed; the commits arrive on empty[s] and tfull[b] of both CTAs;
// tempty[b] (CTA 0) takes one arrival from each epilogue warp of both CTAs.
// ---------------------------------------------------------------------------
constexpr int kPM = 128;   // rows per CTA (256 per pair)
constexpr int kPN = 256;   // output columns per pair tile (128 B rows per CTA)
constexpr int kPSmemLimit = 232448;

template <typename OutT>
struct PCfg {
    static constexpr int kABytes = kPM * kGK;
    static constexpr int kBBytes = (kPN / 2) * kGK;
    static constexpr int kStageBytes = kABytes + kBBytes;  // 32 KB
    static constexpr int kStgBytes = kGEpi * 32 * stage_pitch<OutT>();
    static constexpr int kTabBytes = kPN * 4;              // bias of the tile's columns
    static constexpr int kFixed = kStgBytes + kTabBytes + 512 + 1024;
    static constexpr int kFit = (kPSmemLimit - kFixed) / kStageBytes;
    static constexpr int S = kFit > 6 ? 6 : kFit;
    static_assert(S >= 4, "shared memory budget");
    static constexpr int kStgOff = S * kStageBytes;
    static constexpr int kTabOff = kStgOff + kStgBytes;
    static constexpr int kBarOff = kTabOff + kTabBytes;
    static constexpr int kTotal = kBarOff + 512 + 1024;
    static_assert((2 * S + 4) * 8 + 4 <= 512, "barrier area");
    static constexpr uint32_t kAccCols = kPN;
    static constexpr uint32_t kTmemCols = 2 * kAccCols;
};

__device__ __forceinline__ void mma_f8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The work of pair p: the whole tiles p, p + np, ... below t_full; then, when
// the last wave of tiles is split (rem > 0), half of the contraction of
// remainder tile t_full + p / 2 (pairs p < 2 rem), whose raw fp32
// accumulator goes to part[tile - t_full][half] for fp8_combine_kernel.
struct PairUnits {
    int t_full, rem, nkb, p, np;
    __device__ int whole() const { return p < t_full ? (t_full - 1 - p) / np + 1 : 0; }
    __device__ int count() const { return whole() + (p < 2 * rem ? 1 : 0); }
    __device__ void get(int u, int& t, int& kb0, int& kb1, int& half) const {
        if (u < whole()) {
            t = p + u * np;
            kb0 = 0;
            kb1 = nkb;
            half = -1;
        } else {
            t = t_full + p / 2;
            half = p % 2;
            kb0 = half ? nkb / 2 : 0;
            kb1 = half ? nkb : nkb / 2;
        }
    }
};

template <typename OutT>
__global__ void __launch_bounds__(kGThreads, 1)
    fp8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         int M, int N, int K, uint32_t idesc, const float* __restrict__ sa,
                         const float* __restrict__ sb, const float* __restrict__ bias, OutT* __restrict__ C,
                         int t_full, int rem, float* __restrict__ part, int* status) {
    using P = PCfg<OutT>;
    constexpr int S = P::S;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + P::kBarOff);  // [S] (CTA 0)
    uint64_t* empty = full + S;                                       // [S]
    uint64_t* tfull = empty + S;                                      // [2]
    uint64_t* tempty = tfull + 2;                                     // [2] (CTA 0)
    uint32_t* tslot = reinterpret_cast<uint32_t*>(tempty + 2);
    float* sBias = reinterpret_cast<float*>(smem + P::kTabOff);

    const uint32_t rank = cluster_ctarank();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int pair = static_cast<int>(blockIdx.x) / 2;
    const int npairs = static_cast<int>(gridDim.x) / 2;
    const int num_nt = (N + kPN - 1) / kPN;
    const int nkb = (K + kGK - 1) / kGK;
    const PairUnits U{t_full, rem, nkb, pair, npairs};
    const int nunits = U.count();
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 2 * kGEpi);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tslot, P::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    // neither CTA signals the other's barriers before both have initialised them
    cluster_arrive();
    cluster_wait();
    pdl_wait();  // nothing above touched global memory

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            const uint32_t full0 = dsmem_addr(full, 0);  // CTA 0's full[0]
            int g = 0;
            bool ok = true;
            for (int u = 0; u < nunits && ok; ++u) {
                int t, kb0, kb1, half;
                U.get(u, t, kb0, kb1, half);
                const int m0 = (t / num_nt) * 2 * kPM + static_cast<int>(rank) * kPM;
                const int n0 = (t % num_nt) * kPN + static_cast<int>(rank) * (kPN / 2);
                for (int kb = kb0; kb < kb1; ++kb, ++g) {
                    const int s = g % S;
                    if (g >= S && !mbar_wait(&empty[s], ((g / S) - 1) & 1, status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + s * P::kStageBytes;
                    if (rank == 0) {
                        mbar_arrive_expect_tx(&full[s], 2 * P::kStageBytes);
                        tma_load_2d(st, &tmA, &full[s], kb * kGK, m0);
                        tma_load_2d(st + P::kABytes, &tmB, &full[s], kb * kGK, n0);
                    } else {
                        const uint32_t fb = full0 + 8u * static_cast<uint32_t>(s);
                        tma_load_2d_pair(st, &tmA, fb, kb * kGK, m0);
                        tma_load_2d_pair(st + P::kABytes, &tmB, fb, kb * kGK, n0);
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer (CTA 0)
        if (rank == 0 && lane == 0) {
            int g = 0, i = 0;
            bool ok = true;
            for (int u = 0; u < nunits && ok; ++u, ++i) {
                int t, kb0, kb1, half;
                U.get(u, t, kb0, kb1, half);
                const int ab = i & 1;
                const int use = i >> 1;
                if (use > 0 && !mbar_wait(&tempty[ab], (use - 1) & 1, status)) break;
                tc_fence_after();
                const uint32_t dacc = tmem + ab * P::kAccCols;
                for (int kb = kb0; kb < kb1; ++kb, ++g) {
                    const int s = g % S;
                    if (!mbar_wait(&full[s], (g / S) & 1, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + s * P::kStageBytes);
                    const uint32_t b_base = a_base + P::kABytes;
#pragma unroll
                    for (int kk = 0; kk < kGK / 32; ++kk) {
                        const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024, kLayoutSw128);
                        const uint64_t bd = smem_desc(b_base + kk * 32, 16, 1024, kLayoutSw128);
                        mma_f8_pair(dacc, ad, bd, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
                    }
                    mma_commit_pair(&empty[s], 0x3);
                }
                if (ok) mma_commit_pair(&tfull[ab], 0x3);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int ew = warp - 2;  // 0 .. 3
        const int q = warp & 3;   // TMEM lane quarter of this warp
        const int et = threadIdx.x - 64;
        uint8_t* stg = smem + P::kStgOff + ew * 32 * stage_pitch<OutT>();
        const bool vec = ((static_cast<size_t>(N) * sizeof(OutT)) % 16) == 0;
        const uint32_t tempty0 = dsmem_addr(tempty, 0);
        const float sab = __fmul_rn(__ldg(sa), __ldg(sb));
        int i = 0;
        for (int u = 0; u < nunits; ++u, ++i) {
            int t, kb0, kb1, half;
            U.get(u, t, kb0, kb1, half);
            const int ab = i & 1;
            const int use = i >> 1;
            const int m0 = (t / num_nt) * 2 * kPM + static_cast<int>(rank) * kPM;
            const int n0 = (t % num_nt) * kPN;
            // the tile's bias (the last tile's reads are done)
            named_bar_sync(1, 32 * kGEpi);
            for (int col = et; col < kPN; col += 32 * kGEpi) {
                const int n = n0 + col;
                sBias[col] = (bias && n < N) ? __ldg(bias + n) : 0.f;
            }
            named_bar_sync(1, 32 * kGEpi);
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[ab], use & 1, status));
            if (!ok) break;
            tc_fence_after();
            const int row0 = m0 + q * 32;
            const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + ab * P::kAccCols;
            if (half >= 0) {
                // half of a split tile: the raw accumulator, row-major over the
                // pair's 256 rows, for fp8_combine_kernel
                float* dst = part + (static_cast<size_t>(t - t_full) * 2 + half) * (2 * kPM * kPN) +
                             static_cast<size_t>(static_cast<int>(rank) * kPM + q * 32 + lane) * kPN;
#pragma unroll 1
                for (int col = 0; col < kPN; col += kEpiCols) {
                    uint32_t v[kEpiCols];
                    tmem_ld16(tbase + col, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < kEpiCols; e += 4)
                        *reinterpret_cast<uint4*>(dst + col + e) = make_uint4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                }
            } else if (nkb > 0) {
#pragma unroll 1
                for (int col = 0; col < kPN; col += kEpiCols) {
                    uint32_t v[kEpiCols];
                    tmem_ld16(tbase + col, v);
                    tmem_ld_wait();
                    float y[kEpiCols];
#pragma unroll
                    for (int e = 0; e < kEpiCols; ++e) y[e] = fmaf(__uint_as_float(v[e]), sab, sBias[col + e]);
                    store_block<OutT>(stg, y, lane, C, static_cast<size_t>(N), row0, M, n0 + col, N, vec);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) mbar_arrive(&tempty[ab]);
                else mbar_arrive_remote_cta(tempty0 + 8u * static_cast<uint32_t>(ab));
            }
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    // both CTAs are done with the pair's TMEM and with each other's barriers
    cluster_arrive();
    cluster_wait();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, P::kTmemCols);
    }
}

// The split tiles: C = (P0 + P1) sa sb + bias over each tile's 256 x 256
// elements inside the matrix (the sum of the two halves' fp32 accumulators,
// the same in either order).
template <typename OutT>
__global__ void __launch_bounds__(256) fp8_combine_kernel(const float* __restrict__ part, int rem, int t_full,
                                                         int num_nt, int M, int N, const float* __restrict__ sa,
                                                         const float* __restrict__ sb,
                                                         const float* __restrict__ bias, OutT* __restrict__ C) {
    pdl_trigger();
    pdl_wait();
    const float sab = __fmul_rn(__ldg(sa), __ldg(sb));
    constexpr int kTileElems = 2 * kPM * kPN;
    const size_t total = static_cast<size_t>(rem) * (kTileElems / 4);
    for (size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const size_t e = idx * 4;
        const int tl = static_cast<int>(e / kTileElems);
        const int w = static_cast<int>(e % kTileElems);
        const int row = w / kPN, col = w % kPN;
        const int t = t_full + tl;
        const int m = (t / num_nt) * 2 * kPM + row;
        const int n0 = (t % num_nt) * kPN + col;
        if (m >= M || n0 >= N) continue;
        const float4 a = __ldg(reinterpret_cast<const float4*>(part + static_cast<size_t>(tl) * 2 * kTileElems + w));
        const float4 b =
            __ldg(reinterpret_cast<const float4*>(part + (static_cast<size_t>(tl) * 2 + 1) * kTileElems + w));
        const float acc[4] = {a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + j;
            if (n < N)
                C[static_cast<size_t>(m) * N + n] = ActIO<OutT>::from_f(fmaf(acc[j], sab, bias ? __ldg(bias + n) : 0.f));
        }
    }
}
}  // namespace

bool fp8_tiled_applies(const void* T, int R, int Cc, const uint8_t* q, const uint8_t* qt) {
    const auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; };
    return al(T, 16) && Cc % 8 == 0 && al(q, 8) && (!qt || (al(qt, 16) && R % 16 == 0)) &&
           (Cc + kFC - 1) / kFC <= 65535;
}

// workspace: the amax word; with column sums, from byte 256 the partial sums
// [row tiles][Cc]
static size_t colsum_part_offset(int) { return 256; }

size_t fp8_colsum_ws_bytes(int R, int Cc) {
    return colsum_part_offset(Cc) + 4 * static_cast<size_t>((R + kFR - 1) / kFR) * static_cast<size_t>(Cc);
}

cudaError_t launch_fp8_quantize(Act act, const void* T, int R, int Cc, const float* scale_in, float* scale_out,
                                float* hist, int L, int fmt, uint8_t* q, uint8_t* qt, void* ws, float* colsum,
                                cudaStream_t s) {
    unsigned int* amax_word = static_cast<unsigned int*>(ws);
    float* part = colsum ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + colsum_part_offset(Cc)) : nullptr;
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(unsigned int), s);
    if (e != cudaSuccess) return e;
    const bool tiled = fp8_tiled_applies(T, R, Cc, q, qt);
    if (colsum && !tiled) return cudaErrorInvalidValue;
    if (tiled) {
        const dim3 grid((R + kFR - 1) / kFR, (Cc + kFC - 1) / kFC);
        auto go = [&](auto kern, auto src) {
            return launch_k(kern, grid, dim3(kFThreads), 0, s, 1, src, R, Cc, scale_in, q, qt, amax_word, part);
        };
        const auto* sb = static_cast<const __nv_bfloat16*>(T);
        const auto* sf = static_cast<const float*>(T);
        const bool e4 = fmt == kFp8E4M3;
        if (colsum) {
            if (act == kBF16)
                e = e4 ? go(fp8_quantize_tiled_kernel<__nv_bfloat16, kFp8E4M3, true>, sb)
                       : go(fp8_quantize_tiled_kernel<__nv_bfloat16, kFp8E5M2, true>, sb);
            else
                e = e4 ? go(fp8_quantize_tiled_kernel<float, kFp8E4M3, true>, sf)
                       : go(fp8_quantize_tiled_kernel<float, kFp8E5M2, true>, sf);
        } else {
            if (act == kBF16)
                e = e4 ? go(fp8_quantize_tiled_kernel<__nv_bfloat16, kFp8E4M3, false>, sb)
                       : go(fp8_quantize_tiled_kernel<__nv_bfloat16, kFp8E5M2, false>, sb);
            else
                e = e4 ? go(fp8_quantize_tiled_kernel<float, kFp8E4M3, false>, sf)
                       : go(fp8_quantize_tiled_kernel<float, kFp8E5M2, false>, sf);
        }
    } else {
        if ((Cc + kQT - 1) / kQT > 65535) return cudaErrorInvalidValue;
        const dim3 grid((R + kQT - 1) / kQT, (Cc + kQT - 1) / kQT);
        e = act == kBF16
                ? launch_k(fp8_quantize_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, 1,
                           static_cast<const __nv_bfloat16*>(T), R, Cc, scale_in, fmt, q, qt, amax_word)
                : launch_k(fp8_quantize_kernel<float>, grid, dim3(256), 0, s, 1, static_cast<const float*>(T), R,
                           Cc, scale_in, fmt, q, qt, amax_word);
    }
    if (e != cudaSuccess) return e;
    if (colsum) {
        e = launch_k(fp8_colsum_kernel, dim3((Cc + kCsCols - 1) / kCsCols), dim3(32 * kCsWarps), 0, s, 1,
                     static_cast<const float*>(part), (R + kFR - 1) / kFR, Cc, colsum);
        if (e != cudaSuccess) return e;
    }
    const float fmax = fmt == kFp8E4M3 ? 448.0f : 57344.0f;
    return launch_k(fp8_state_kernel, dim3(1), dim3(1024), 0, s, 1, static_cast<const unsigned int*>(amax_word),
                    scale_in, scale_out, hist, L, fmax);
}

// Split of the pairs' last wave of tiles: with T pair tiles on np pairs, rem =
// T mod np tiles left for a partial last wave are computed as two halves of
// the contraction each (2 rem <= np half-tiles, one wave of half the length)
// when a workspace holds their partials.  Returns the rem used (0: none).
static int fp8_split_rem(int M, int N, int K) {
    const long long tiles =
        static_cast<long long>((M + 2 * kPM - 1) / (2 * kPM)) * ((N + kPN - 1) / kPN);
    const int np = sm_count() / 2;
    if (tiles < np || (K + kGK - 1) / kGK < 2) return 0;
    const int rem = static_cast<int>(tiles % np);
    return (rem > 0 && 2 * rem <= np) ? rem : 0;
}

size_t fp8_gemm_ws_bytes(int M, int N, int K) {
    return static_cast<size_t>(fp8_split_rem(M, N, K)) * 2 * (2 * kPM * kPN) * sizeof(float);
}

cudaError_t launch_fp8_gemm(const uint8_t* A, int afmt, const uint8_t* B, int bfmt, int M, int N, int K,
                            const float* sa, const float* sb, const float* bias, void* C, Act out, int* status,
                            cudaStream_t s, void* ws, size_t ws_bytes) {
    CUtensorMap ta, tb;
    if (!make_tmap_2d(&ta, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K, K, kGM, kGK, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tb, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, K, 128, kGK, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int bn = N >= 256 ? 256 : 128;
    CUtensorMap tb2;
    if (!make_tmap_2d(&tb2, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, K, bn, kGK, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int pair_tiles = ((M + 2 * kPM - 1) / (2 * kPM)) * ((N + kPN - 1) / kPN);
    if (pair_tiles >= sm_count() / 2) {
        // CTA pairs, persistent: one pair per two SMs; tb holds 128-row boxes of B
        const int pairs = pair_tiles < sm_count() / 2 ? pair_tiles : sm_count() / 2;
        const uint32_t idp = idesc_f8(2 * kPM, kPN, afmt, bfmt);
        // the last wave split in halves where a workspace holds the partials
        const size_t need = fp8_gemm_ws_bytes(M, N, K);
        const int rem = (need > 0 && ws && ws_bytes >= need) ? fp8_split_rem(M, N, K) : 0;
        const int t_full = rem ? pair_tiles - rem : pair_tiles;
        float* part = rem ? static_cast<float*>(ws) : nullptr;
        auto runp = [&](auto kern, int total) -> cudaError_t {
            cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), total);
            if (e != cudaSuccess) return e;
            return launch_kx(kern, dim3(2 * pairs), dim3(kGThreads), static_cast<size_t>(total), s, 2, ta, tb, M,
                             N, K, idp, sa, sb, bias, C, t_full, rem, part, status);
        };
        const int num_nt = (N + kPN - 1) / kPN;
        const int cgrid = rem * (2 * kPM * kPN / 4) / 256;
        cudaError_t e;
        if (out == kBF16) {
            e = runp(fp8_gemm_pair_kernel<__nv_bfloat16>, PCfg<__nv_bfloat16>::kTotal);
            if (e == cudaSuccess && rem)
                e = launch_k(fp8_combine_kernel<__nv_bfloat16>, dim3(cgrid), dim3(256), 0, s, 1,
                             static_cast<const float*>(part), rem, t_full, num_nt, M, N, sa, sb, bias,
                             static_cast<__nv_bfloat16*>(C));
        } else {
            e = runp(fp8_gemm_pair_kernel<float>, PCfg<float>::kTotal);
            if (e == cudaSuccess && rem)
                e = launch_k(fp8_combine_kernel<float>, dim3(cgrid), dim3(256), 0, s, 1,
                             static_cast<const float*>(part), rem, t_full, num_nt, M, N, sa, sb, bias,
                             static_cast<float*>(C));
        }
        return e;
    }
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
