// k1_quantize.cu -- per-row abs-max int8 quantization of the layer input,
// fused with the LoRA down-projection x . A, and the one-off per-output-
// channel quantization of the frozen kernel.
//
// The quantizer ("Introduce QLoRA-like technique": frozen int8 Dense with
// dynamically quantized inputs) is symmetric abs-max in IEEE fp32 with one
// rounding per operation: inv = 127 / amax, q = clamp(rne(v * inv), -127,
// 127), s = amax / 127.  The LoRA term uses the unquantized input
// ("Parameter-efficient fine-tuning of GPT-2 with LoRA", "LoRA equation").
//
// K1 is HBM-bound: it reads M*K*e bytes of X once (128-bit loads held in
// registers), writes M*K int8 codes, M scales and M*r floats of xA.  The
// LoRA factor A [K,r] is staged in shared memory once per CTA (padded so that
// the 8-row slices the lanes read are bank-conflict free) and the CTA then
// walks over many row groups, so A is read from L2 once per CTA, not per row.
#include "internal.h"
#include "ptx.cuh"
#include "tile_epilogue.cuh"

namespace qlora {

namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 8;    // elements per 128-bit (bf16) / 2x128-bit (f32) load
constexpr int kMaxCPT = 8;   // chunks per thread held in registers
constexpr int kSmemCap = 200 * 1024;
constexpr int kSlicedSmem = 96 * 1024;  // A slice of the sliced kernel: two CTAs per SM

template <typename T>
struct Chunk8;

template <>
struct Chunk8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
        uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(h[i]);
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
};

template <>
struct Chunk8<float> {
    static __device__ __forceinline__ void load(const float* p, float (&v)[8]) {
        float4 a = __ldg(reinterpret_cast<const float4*>(p));
        float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

__device__ __forceinline__ uint2 pack8(const float (&v)[8], float inv) {
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) lo |= (static_cast<uint32_t>(quant_code(v[i], inv)) & 0xFFu) << (8 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i) hi |= (static_cast<uint32_t>(quant_code(v[4 + i], inv)) & 0xFFu) << (8 * i);
    return make_uint2(lo, hi);
}

// Floats of the staged A slice for `chunks` 8-row chunks: each chunk holds
// 8 rows of RP floats followed by 4 floats of padding.
template <int RP>
__host__ __device__ constexpr int a_chunk_floats() { return 8 * RP + 4; }

// Stages A rows [k0, k0 + 8*chunks) into shared memory (zero outside K / r).
// Every round issues all its loads (from addresses clamped into A) before
// any of them is used, so a round costs one memory latency; a select on each
// freshly loaded value would wait out the loads one by one.
template <int RP>
__device__ __forceinline__ void stage_a(float* sA, const float* __restrict__ A, int K, int r,
                                        int k0, int chunks) {
    constexpr int kU = 8;  // loads in flight per thread
    if (r == RP && (reinterpret_cast<uintptr_t>(A) & 15) == 0) {
        // rows of A are RP floats: copy 16-byte vectors
        constexpr int V = 2 * RP;  // float4 per 8-row chunk
        const int n4 = chunks * V;
        const int kmax4 = (K - k0) * RP / 4;  // float4 that lie inside A
        const int lim = n4 < kmax4 ? n4 : kmax4;
        const float4* src = reinterpret_cast<const float4*>(A + static_cast<size_t>(k0) * RP);
        float4* dst = reinterpret_cast<float4*>(sA);
        for (int base = threadIdx.x; base < n4; base += kU * blockDim.x) {
            float4 v[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int idx = base + u * blockDim.x;
                v[u] = __ldg(src + (idx < lim ? idx : lim - 1));
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int idx = base + u * blockDim.x;
                if (idx < n4)
                    dst[(idx / V) * (V + 1) + idx % V] = idx < lim ? v[u] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        return;
    }
    const int n = chunks * 8 * RP;
    for (int base = threadIdx.x; base < n; base += kU * blockDim.x) {
        float v[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int idx = base + u * blockDim.x;
            const int kl = idx / RP, j = idx % RP;
            const int k = k0 + kl < K ? k0 + kl : K - 1;
            v[u] = __ldg(A + static_cast<size_t>(k) * r + (j < r ? j : r - 1));
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int idx = base + u * blockDim.x;
            const int kl = idx / RP, j = idx % RP;
            if (idx < n)
                sA[(kl >> 3) * a_chunk_floats<RP>() + (kl & 7) * RP + j] =
                    (k0 + kl < K && j < r) ? v[u] : 0.f;
        }
    }
}

// acc[j] += sum_e v[e] * A[chunk row e, j] with the chunk's rows in shared memory.
template <int RP>
__device__ __forceinline__ void chunk_fma(const float* sA_chunk, const float (&v)[8],
                                          float (&acc)[RP]) {
    const float4* a4 = reinterpret_cast<const float4*>(sA_chunk);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
#pragma unroll
        for (int j4 = 0; j4 < RP / 4; ++j4) {
            const float4 a = a4[e * (RP / 4) + j4];
            acc[4 * j4 + 0] = fmaf(v[e], a.x, acc[4 * j4 + 0]);
            acc[4 * j4 + 1] = fmaf(v[e], a.y, acc[4 * j4 + 1]);
            acc[4 * j4 + 2] = fmaf(v[e], a.z, acc[4 * j4 + 2]);
            acc[4 * j4 + 3] = fmaf(v[e], a.w, acc[4 * j4 + 3]);
        }
    }
}

// Sum (or max) over the TPR threads that share a row (TPR in {32,64,128,256}).
// `red` holds kThreads/32 floats per call site.
template <int TPR, bool IS_MAX>
__device__ __forceinline__ float row_reduce(float v, float* red, int row_in_block, int t) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        float w = __shfl_xor_sync(0xffffffffu, v, o);
        v = IS_MAX ? fmaxf(v, w) : v + w;
    }
    if constexpr (TPR > 32) {
        constexpr int W = TPR / 32;
        if ((t & 31) == 0) red[row_in_block * W + (t >> 5)] = v;
        __syncthreads();
        float s = red[row_in_block * W];
#pragma unroll
        for (int i = 1; i < W; ++i) {
            float w = red[row_in_block * W + i];
            s = IS_MAX ? fmaxf(s, w) : s + w;
        }
        __syncthreads();
        v = s;
    }
    return v;
}

// TPR threads per row, 256/TPR rows per group; the CTA walks row groups
// blockIdx.x, blockIdx.x + gridDim.x, ...  A is staged once if it fits
// (a_chunks >= number of chunks of a row), else in slices of a_chunks.
template <typename T, int TPR, int RP>
__global__ void __launch_bounds__(kThreads) k1_quantize_rows_kernel(
    const T* __restrict__ X, const float* __restrict__ A, int M, int K, int r, int a_chunks,
    int8_t* __restrict__ Xq, float* __restrict__ sx, float* __restrict__ xA) {
    constexpr int RPB = kThreads / TPR;
    pdl_trigger();
    pdl_wait();
    extern __shared__ float4 smem_f4[];
    float* sA = reinterpret_cast<float*>(smem_f4);
    __shared__ float red[kThreads / 32];
    const int row_in_block = threadIdx.x / TPR;
    const int t = threadIdx.x % TPR;
    const int nchunks = K / kChunk;
    const int groups = (M + RPB - 1) / RPB;
    const bool whole_a = a_chunks >= nchunks;
    bool staged = false;

    for (int grp = blockIdx.x; grp < groups; grp += gridDim.x) {
        const int m = grp * RPB + row_in_block;
        const bool live = m < M;
        const T* xr = X + static_cast<size_t>(live ? m : 0) * K;

        // the row's loads go out first; A is staged while they are in flight
        float v[kMaxCPT][8];
#pragma unroll
        for (int i = 0; i < kMaxCPT; ++i) {
            const int ch = t + i * TPR;
            if (live && ch < nchunks) {
                Chunk8<T>::load(xr + ch * kChunk, v[i]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) v[i][e] = 0.f;
            }
        }
        if (whole_a && !staged) {
            stage_a<RP>(sA, A, K, r, 0, nchunks);
            __syncthreads();
            staged = true;
        }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxCPT; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[i][e]));
        amax = row_reduce<TPR, true>(amax, red, row_in_block, t);
        const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
        if (live) {
            int8_t* qr = Xq + static_cast<size_t>(m) * K;
#pragma unroll
            for (int i = 0; i < kMaxCPT; ++i) {
                const int ch = t + i * TPR;
                if (ch < nchunks) *reinterpret_cast<uint2*>(qr + ch * kChunk) = pack8(v[i], inv);
            }
            if (t == 0) sx[m] = __fdiv_rn(amax, 127.0f);
        }

        // xA[m, :] = X[m, :] . A
        float acc[RP];
#pragma unroll
        for (int j = 0; j < RP; ++j) acc[j] = 0.f;
        if (whole_a) {
#pragma unroll
            for (int i = 0; i < kMaxCPT; ++i) {
                const int ch = t + i * TPR;
                if (live && ch < nchunks) chunk_fma<RP>(sA + ch * a_chunk_floats<RP>(), v[i], acc);
            }
        } else {
            for (int c0 = 0; c0 < nchunks; c0 += a_chunks) {
                __syncthreads();
                stage_a<RP>(sA, A, K, r, c0 * kChunk, a_chunks);
                __syncthreads();
#pragma unroll
                for (int i = 0; i < kMaxCPT; ++i) {
                    const int ch = t + i * TPR;
                    if (live && ch < nchunks && ch >= c0 && ch < c0 + a_chunks)
                        chunk_fma<RP>(sA + (ch - c0) * a_chunk_floats<RP>(), v[i], acc);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < RP; ++j) {
            const float s = row_reduce<TPR, false>(acc[j], red, row_in_block, t);
            if (live && t == 0 && j < r) xA[static_cast<size_t>(m) * r + j] = s;
        }
    }
}

// Rows longer than 256*64 elements: one CTA per row, two sweeps over global
// memory (abs-max, then quantize + x.A), A staged in slices.
template <typename T, int RP>
__global__ void __launch_bounds__(kThreads) k1_quantize_rows_long_kernel(
    const T* __restrict__ X, const float* __restrict__ A, int M, int K, int r, int a_chunks,
    int8_t* __restrict__ Xq, float* __restrict__ sx, float* __restrict__ xA) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ float4 smem_f4[];
    float* sA = reinterpret_cast<float*>(smem_f4);
    __shared__ float red[kThreads / 32];
    const int m = blockIdx.x;
    const int t = threadIdx.x;
    const int nchunks = K / kChunk;
    const T* xr = X + static_cast<size_t>(m) * K;
    float amax = 0.f;
    for (int ch = t; ch < nchunks; ch += kThreads) {
        float v[8];
        Chunk8<T>::load(xr + ch * kChunk, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
    }
    amax = row_reduce<kThreads, true>(amax, red, 0, t);
    const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
    int8_t* qr = Xq + static_cast<size_t>(m) * K;
    float acc[RP];
#pragma unroll
    for (int j = 0; j < RP; ++j) acc[j] = 0.f;
    for (int c0 = 0; c0 < nchunks; c0 += a_chunks) {
        __syncthreads();
        stage_a<RP>(sA, A, K, r, c0 * kChunk, a_chunks);
        __syncthreads();
        for (int ch = c0 + t; ch < c0 + a_chunks && ch < nchunks; ch += kThreads) {
            float v[8];
            Chunk8<T>::load(xr + ch * kChunk, v);
            *reinterpret_cast<uint2*>(qr + ch * kChunk) = pack8(v, inv);
            chunk_fma<RP>(sA + (ch - c0) * a_chunk_floats<RP>(), v, acc);
        }
    }
    if (t == 0) sx[m] = __fdiv_rn(amax, 127.0f);
#pragma unroll
    for (int j = 0; j < RP; ++j) {
        const float s = row_reduce<kThreads, false>(acc[j], red, 0, t);
        if (t == 0 && j < r) xA[static_cast<size_t>(m) * r + j] = s;
    }
}

// Rows whose x.A operand A does not fit in shared memory.  A CTA takes 32
// rows, four per warp, and sweeps them twice: the abs-max of each row, then,
// A slice by A slice (each slice staged once for all 32 rows instead of once
// per row), the quantization of the slice's chunks and their part of x.A.
// Eight 8-element chunks of a row are loaded before any is used, and the A
// slices are sized for two CTAs per SM, so that enough bytes are in flight
// per SM to cover the memory latency.
template <typename T, int RP>
__global__ void __launch_bounds__(kThreads) k1_quantize_rows_sliced_kernel(
    const T* __restrict__ X, const float* __restrict__ A, int M, int K, int r, int a_chunks,
    int8_t* __restrict__ Xq, float* __restrict__ sx, float* __restrict__ xA) {
    constexpr int kRowsPerWarp = 4;
    constexpr int kRows = kRowsPerWarp * (kThreads / 32);
    constexpr int kU = 8;
    pdl_trigger();
    pdl_wait();
    extern __shared__ float4 smem_f4[];
    float* sA = reinterpret_cast<float*>(smem_f4);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nchunks = K / kChunk;
    const int m0 = blockIdx.x * kRows + warp * kRowsPerWarp;
    float inv[kRowsPerWarp];
#pragma unroll
    for (int q = 0; q < kRowsPerWarp; ++q) {
        const int m = m0 + q;
        float amax = 0.f;
        if (m < M) {
            const T* xr = X + static_cast<size_t>(m) * K;
            for (int ch = lane; ch < nchunks; ch += 32 * kU) {
                float v[kU][8];
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int c = ch + 32 * u;
                    Chunk8<T>::load(xr + static_cast<size_t>(c < nchunks ? c : nchunks - 1) * kChunk, v[u]);
                }
#pragma unroll
                for (int u = 0; u < kU; ++u)
                    if (ch + 32 * u < nchunks)
#pragma unroll
                        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[u][e]));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        inv[q] = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
        if (m < M && lane == 0) sx[m] = __fdiv_rn(amax, 127.0f);
    }
    float acc[kRowsPerWarp][RP];
#pragma unroll
    for (int q = 0; q < kRowsPerWarp; ++q)
#pragma unroll
        for (int j = 0; j < RP; ++j) acc[q][j] = 0.f;
    for (int c0 = 0; c0 < nchunks; c0 += a_chunks) {
        const int c1 = c0 + a_chunks < nchunks ? c0 + a_chunks : nchunks;
        __syncthreads();  // the previous slice is no longer read
        stage_a<RP>(sA, A, K, r, c0 * kChunk, c1 - c0);
        __syncthreads();
#pragma unroll
        for (int q = 0; q < kRowsPerWarp; ++q) {
            const int m = m0 + q;
            if (m >= M) continue;  // warp-uniform
            const T* xr = X + static_cast<size_t>(m) * K;
            int8_t* qr = Xq + static_cast<size_t>(m) * K;
            for (int ch = c0 + lane; ch < c1; ch += 32 * kU) {
                float v[kU][8];
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int c = ch + 32 * u;
                    Chunk8<T>::load(xr + static_cast<size_t>(c < c1 ? c : c1 - 1) * kChunk, v[u]);
                }
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int c = ch + 32 * u;
                    if (c < c1) {
                        *reinterpret_cast<uint2*>(qr + static_cast<size_t>(c) * kChunk) = pack8(v[u], inv[q]);
                        chunk_fma<RP>(sA + (c - c0) * a_chunk_floats<RP>(), v[u], acc[q]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int q = 0; q < kRowsPerWarp; ++q) {
        const int m = m0 + q;
#pragma unroll
        for (int j = 0; j < RP; ++j) {
            float v = acc[q][j];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (m < M && lane == 0 && j < r) xA[static_cast<size_t>(m) * r + j] = v;
        }
    }
}

template <typename T, int RP>
cudaError_t launch_sliced(const T* X, const float* A, int M, int K, int r, int8_t* Xq, float* sx,
                          float* xA, cudaStream_t s) {
    const int nchunks = K / kChunk;
    const int cap_chunks = kSlicedSmem / (a_chunk_floats<RP>() * 4);
    const int a_chunks = nchunks <= cap_chunks ? nchunks : cap_chunks;
    auto kern = k1_quantize_rows_sliced_kernel<T, RP>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), kSmemCap);
    if (e != cudaSuccess) return e;
    constexpr int kRows = 4 * (kThreads / 32);
    return launch_k(kern, dim3((M + kRows - 1) / kRows), dim3(kThreads),
                    a_chunks * a_chunk_floats<RP>() * 4, s, 1, X, A, M, K, r, a_chunks, Xq, sx, xA);
}

template <typename T, int TPR, int RP>
cudaError_t launch_tpr(const T* X, const float* A, int M, int K, int r, int8_t* Xq, float* sx,
                       float* xA, cudaStream_t s) {
    const int nchunks = K / kChunk;
    const int cap_chunks = kSmemCap / (a_chunk_floats<RP>() * 4);
    const int a_chunks = nchunks <= cap_chunks ? nchunks : cap_chunks;
    const int smem = a_chunks * a_chunk_floats<RP>() * 4;
    auto kern = k1_quantize_rows_kernel<T, TPR, RP>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), kSmemCap);
    if (e != cudaSuccess) return e;
    constexpr int RPB = kThreads / TPR;
    const int groups = (M + RPB - 1) / RPB;
    // whole A staged once: persistent over row groups; else one group per CTA
    const int per_sm = smem <= 48 * 1024 ? 4 : (smem <= 100 * 1024 ? 2 : 1);
    int grid = groups;
    if (a_chunks >= nchunks && grid > per_sm * sm_count()) grid = per_sm * sm_count();
    return launch_k(kern, dim3(grid), dim3(kThreads), smem, s, 1, X, A, M, K, r, a_chunks, Xq, sx, xA);
}

template <typename T, int RP>
cudaError_t launch_rows_rp(const T* X, const float* A, int M, int K, int r, int8_t* Xq, float* sx,
                           float* xA, cudaStream_t s) {
    const int nchunks = K / kChunk;
    // A too large for shared memory: slices staged once per 32 rows
    if constexpr (RP <= 16) {
        if (nchunks > kSmemCap / (a_chunk_floats<RP>() * 4))
            return launch_sliced<T, RP>(X, A, M, K, r, Xq, sx, xA, s);
    }
    if (nchunks <= 32 * kMaxCPT) return launch_tpr<T, 32, RP>(X, A, M, K, r, Xq, sx, xA, s);
    if (nchunks <= 64 * kMaxCPT) return launch_tpr<T, 64, RP>(X, A, M, K, r, Xq, sx, xA, s);
    if (nchunks <= 128 * kMaxCPT) return launch_tpr<T, 128, RP>(X, A, M, K, r, Xq, sx, xA, s);
    if (nchunks <= 256 * kMaxCPT) return launch_tpr<T, 256, RP>(X, A, M, K, r, Xq, sx, xA, s);
    const int cap_chunks = kSmemCap / (a_chunk_floats<RP>() * 4);
    const int a_chunks = nchunks <= cap_chunks ? nchunks : cap_chunks;
    auto kern = k1_quantize_rows_long_kernel<T, RP>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), kSmemCap);
    if (e != cudaSuccess) return e;
    return launch_k(kern, dim3(M), dim3(kThreads), a_chunks * a_chunk_floats<RP>() * 4, s, 1, X, A, M,
                    K, r, a_chunks, Xq, sx, xA);
}

// ------------------------------------------------------------------ staged K1
// bf16 rows, rank <= 8, rows of at most 256 * CPT 8-element chunks.
//
// Rows stream through a ring of shared-memory stages, each filled by one
// bulk copy of R consecutive rows (four per row group, up to 32 KB), so that
// a CTA keeps up to five stages (160 KB) of loads in flight with one
// instruction per stage.  Eight consumer warps form row groups of TPR threads
// (TPR a multiple of 32 covering the row); a thread owns one or two 8-element
// chunks of the row and holds the matching rows of A in registers, so x.A
// costs no shared-memory traffic.
// Per stage a row group takes two sweeps over its staged rows: the abs-max,
// then the codes (written as 8-byte stores) and the x.A partial sums, as
// paired fp32 FMAs over neighbouring elements (the two lanes of a pair are
// added at the end).  Both reductions over the group's threads go through a
// transposing warp butterfly (one shuffle per value and lane step) and,
// across warps, one named barrier each.
namespace staged {
// consumer threads: row groups of TPR threads, 256 in all (eight warps: 512,
// at one chunk per thread, measured slower at 16384 x 4096: the per-stage
// reductions over twice the warps cost more than the extra warps hide)
template <int RP>
__host__ __device__ constexpr int max_cons() { return 256; }
template <int TPR, int RP>
__host__ __device__ constexpr int groups() { return max_cons<RP>() / TPR; }
template <int TPR, int RP>
__host__ __device__ constexpr int cons() { return groups<TPR, RP>() * TPR; }
constexpr int kRPG = 4;                 // rows per group per stage
constexpr int kSmemBudget = 160 * 1024;
constexpr int kMaxStages = 8;
}  // namespace staged

struct StagedArgs {
    const __nv_bfloat16* X;
    const float* A;
    int M, K, r;
    int8_t* Xq;
    float* sx;
    float* xA;
    int rows_per_stage;    // R = groups * kRPG
    uint32_t stage_bytes;  // R * K * 2, rounded up to 128
    int nstages;           // ring depth S
    int stages_total;      // ceil(M / R)
};

// 8 bf16 (16 bytes) -> 8 floats (exact)
__device__ __forceinline__ void bf16x8_to_f(const uint4 u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Symmetric abs-max codes of 8 values: rne(fl(v * inv)).  The products are
// rounded to fp32 lane by lane (mul.rn.f32x2: two per instruction, never
// contracted), converted with round-to-nearest-even (cvt.rni.s32.f32, on the
// conversion pipe beside the FMA pipe) and packed four to a word with
// saturation (cvt.pack.sat.s8.s32: |fl(v * inv)| <= 127 * (1 + 2^-24)^2 <
// 127.5, so saturation is never reached).  Against an fp32 multiply, a
// 1.5 * 2^23 add and byte permutes on the FMA pipe this ran 72 against 76 us
// at 16384 x 4096 with the same codes.
__device__ __forceinline__ uint2 codes8(const float (&f)[8], float inv) {
    const unsigned long long inv2 = pk2(inv, inv);
    int c[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        unsigned long long prod;
        asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(prod) : "l"(pk2(f[2 * p], f[2 * p + 1])), "l"(inv2));
        float a, b;
        unpk2(prod, a, b);
        asm("cvt.rni.s32.f32 %0, %1;" : "=r"(c[2 * p]) : "f"(a));
        asm("cvt.rni.s32.f32 %0, %1;" : "=r"(c[2 * p + 1]) : "f"(b));
    }
    uint32_t t0, w0, t1, w1;
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(t0) : "r"(c[3]), "r"(c[2]), "r"(0));
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(w0) : "r"(c[1]), "r"(c[0]), "r"(t0));
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(t1) : "r"(c[7]), "r"(c[6]), "r"(0));
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(w1) : "r"(c[5]), "r"(c[4]), "r"(t1));
    return make_uint2(w0, w1);
}

template <int TPR, int CPT, int RP>
__global__ void __launch_bounds__(staged::cons<TPR, RP>() + 32, 1)
    k1_quantize_rows_staged_kernel(StagedArgs a, int* status) {
    using namespace staged;
    constexpr int kCons = cons<TPR, RP>();
    constexpr int G = groups<TPR, RP>();  // row groups
    constexpr int W = TPR / 32;     // warps per group
    constexpr int V = kRPG * RP;    // x.A partial sums per thread and stage
    static_assert(V <= 32, "transposed reduction width");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
    const int S = a.nstages;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(S) * a.stage_bytes);
    uint64_t* empty = full + kMaxStages;
    float* redA = reinterpret_cast<float*>(empty + kMaxStages);  // [G][kRPG][W]
    float* redX = redA + G * kRPG * W;                           // [G][W][V]
    int* abort_flag = reinterpret_cast<int*>(redX + G * W * V);  // [G]

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int K = a.K;
    const int nch = K >> 3;
    const int R = a.rows_per_stage;
    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kCons / 32);
        }
        for (int g = 0; g < G; ++g) abort_flag[g] = 0;
        fence_mbar_init();
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();

    if (warp == kCons / 32) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int k = 0;
            for (int st = blockIdx.x; st < a.stages_total; st += gridDim.x, ++k) {
                const int slot = k % S;
                if (k >= S && !mbar_wait(&empty[slot], ((k / S) - 1) & 1, status)) break;
                const int row0 = st * R;
                const int rows = min(R, a.M - row0);
                const uint32_t bytes = static_cast<uint32_t>(rows) * static_cast<uint32_t>(K) * 2u;
                mbar_arrive_expect_tx(&full[slot], bytes);
                bulk_load(smem + static_cast<size_t>(slot) * a.stage_bytes,
                          a.X + static_cast<size_t>(row0) * K, bytes, &full[slot]);
            }
            // every copy issued has landed before the CTA may exit
            for (int j = k > S ? k - S : 0; j < k; ++j) mbar_wait(&full[j % S], (j / S) & 1, status);
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    const int g = tid / TPR;
    const int t = tid % TPR;
    const int w = t >> 5;
    // rows of A for this thread's chunks, as (A[k][j], A[k+1][j]) pairs of
    // neighbouring k (k = 8c + 2p)
    unsigned long long a2[CPT][4][RP];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = t + i * TPR;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const int k = c < nch ? c * 8 + 2 * p : 0;
#pragma unroll
            for (int j = 0; j < RP; ++j) {
                const bool in = c < nch && j < a.r;
                const float v0 = in ? __ldg(a.A + static_cast<size_t>(k) * a.r + j) : 0.f;
                const float v1 = in ? __ldg(a.A + static_cast<size_t>(k + 1) * a.r + j) : 0.f;
                a2[i][p][j] = pk2(v0, v1);
            }
        }
    }

    int k = 0;
    for (int st = blockIdx.x; st < a.stages_total; st += gridDim.x, ++k) {
        const int slot = k % S;
        bool ok = mbar_wait(&full[slot], (k / S) & 1, status);
        ok = __all_sync(0xffffffffu, ok);
        const uint8_t* gbase = smem + static_cast<size_t>(slot) * a.stage_bytes +
                               static_cast<size_t>(g * kRPG) * K * 2;
        const int m0 = st * R + g * kRPG;

        // ---- sweep 1: abs-max of each row
        float amax[kRPG];
        float inv[kRPG];  // 127 / amax (0 for a zero row)
#pragma unroll
        for (int q = 0; q < kRPG; ++q) {
            __nv_bfloat162 m2 = __float2bfloat162_rn(0.f);
            if (ok) {
#pragma unroll
                for (int i = 0; i < CPT; ++i) {
                    const int c = t + i * TPR;
                    if (c < nch) {
                        const uint4 u = *reinterpret_cast<const uint4*>(gbase + static_cast<size_t>(q) * K * 2 + c * 16);
                        const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int h = 0; h < 4; ++h)
                            m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&wv[h])));
                    }
                }
            }
            amax[q] = fmaxf(__low2float(m2), __high2float(m2));
        }
        {
            float v[kRPG];
#pragma unroll
            for (int q = 0; q < kRPG; ++q) v[q] = amax[q];
            const float x = xreduce<kRPG, true>(v);
            if constexpr (W == 1) {
#pragma unroll
                for (int q = 0; q < kRPG; ++q) amax[q] = __shfl_sync(0xffffffffu, x, xreduce_lane<kRPG>(q));
#pragma unroll
                for (int q = 0; q < kRPG; ++q) inv[q] = amax[q] > 0.f ? __fdiv_rn(127.0f, amax[q]) : 0.f;
            } else {
                constexpr int kLPR = 32 / kRPG;  // lanes holding one row's value
                const int qr = xreduce_index<kRPG>(lane);
                if ((lane & (kLPR - 1)) == 0) redA[(g * kRPG + qr) * W + w] = x;
                if (!ok) abort_flag[g] = 1;
                named_bar_sync(1 + g, TPR);
                if (abort_flag[g]) break;
                // the kLPR lanes of row qr share its W warp maxima, then every
                // lane takes the four row maxima from one lane of each row
                float mx = 0.f;
#pragma unroll
                for (int ww = lane & (kLPR - 1); ww < W; ww += kLPR)
                    mx = fmaxf(mx, redA[(g * kRPG + qr) * W + ww]);
#pragma unroll
                for (int off = 1; off < kLPR; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
#pragma unroll
                // one division per row, in the row's lanes
                const float iv = mx > 0.f ? __fdiv_rn(127.0f, mx) : 0.f;
#pragma unroll
                for (int q = 0; q < kRPG; ++q) {
                    amax[q] = __shfl_sync(0xffffffffu, mx, xreduce_lane<kRPG>(q));
                    inv[q] = __shfl_sync(0xffffffffu, iv, xreduce_lane<kRPG>(q));
                }
            }
        }
        if (!ok) break;

        // ---- sweep 2: codes and x.A (xa[q][j] holds two partial sums)
        unsigned long long xa[kRPG][RP];
#pragma unroll
        for (int q = 0; q < kRPG; ++q)
#pragma unroll
            for (int j = 0; j < RP; ++j) xa[q][j] = 0ull;
#pragma unroll
        for (int q = 0; q < kRPG; ++q) {
            const int m = m0 + q;
            int8_t* qrow = a.Xq + static_cast<size_t>(m) * K;
#pragma unroll
            for (int i = 0; i < CPT; ++i) {
                const int c = t + i * TPR;
                if (c < nch) {
                    const uint4 u = *reinterpret_cast<const uint4*>(gbase + static_cast<size_t>(q) * K * 2 + c * 16);
                    float f[8];
                    bf16x8_to_f(u, f);
                    const uint2 cw = codes8(f, inv[q]);
                    if (m < a.M) *reinterpret_cast<uint2*>(qrow + c * 8) = cw;
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const unsigned long long x2 = pk2(f[2 * p], f[2 * p + 1]);
#pragma unroll
                        for (int j = 0; j < RP; ++j) fma2(xa[q][j], x2, a2[i][p][j]);
                    }
                }
            }
        }
        // the stage's rows are no longer read: release the slot
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (t < kRPG && m0 + t < a.M) {
            float am = amax[0];
#pragma unroll
            for (int q = 1; q < kRPG; ++q) am = t == q ? amax[q] : am;
            a.sx[m0 + t] = __fdiv_rn(am, 127.0f);
        }

        float v[V];
#pragma unroll
        for (int q = 0; q < kRPG; ++q)
#pragma unroll
            for (int j = 0; j < RP; ++j) {
                float lo, hi;
                unpk2(xa[q][j], lo, hi);
                v[q * RP + j] = lo + hi;
            }
        const float x = xreduce<V, false>(v);
        const int idx = xreduce_index<V>(lane);
        if constexpr (W == 1) {
            if ((lane & (32 / V - 1)) == 0) {
                const int q = idx / RP, j = idx % RP;
                if (m0 + q < a.M && j < a.r) a.xA[static_cast<size_t>(m0 + q) * a.r + j] = x;
            }
        } else {
            if ((lane & (32 / V - 1)) == 0) redX[(g * W + w) * V + idx] = x;
            named_bar_sync(1 + g, TPR);
            if (t < 32) {
                // the group's first warp: 32 / V lanes per value, each adding
                // every (32 / V)-th warp's partial, then a shuffle
                constexpr int kLPV = 32 / V;
                const int vi = t / kLPV;
                float sum = 0.f;
#pragma unroll
                for (int ww = t % kLPV; ww < W; ww += kLPV) sum += redX[(g * W + ww) * V + vi];
#pragma unroll
                for (int off = 1; off < kLPV; off <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                const int q = vi / RP, j = vi % RP;
                if ((t % kLPV) == 0 && m0 + q < a.M && j < a.r) a.xA[static_cast<size_t>(m0 + q) * a.r + j] = sum;
            }
        }
    }
}

template <int TPR, int CPT, int RP>
cudaError_t launch_staged(const __nv_bfloat16* X, const float* A, int M, int K, int r, int8_t* Xq,
                          float* sx, float* xA, int* status, cudaStream_t s) {
    using namespace staged;
    constexpr int G = groups<TPR, RP>();
    constexpr int W = TPR / 32;
    constexpr int V = kRPG * RP;
    StagedArgs a{};
    a.X = X;
    a.A = A;
    a.M = M;
    a.K = K;
    a.r = r;
    a.Xq = Xq;
    a.sx = sx;
    a.xA = xA;
    a.rows_per_stage = G * kRPG;
    a.stage_bytes = (static_cast<uint32_t>(a.rows_per_stage) * K * 2u + 127u) & ~127u;
    int S = kSmemBudget / static_cast<int>(a.stage_bytes);
    S = S > kMaxStages ? kMaxStages : S;
    if (S < 2) return cudaErrorInvalidValue;
    a.nstages = S;
    a.stages_total = (M + a.rows_per_stage - 1) / a.rows_per_stage;
    const size_t smem = 128 + static_cast<size_t>(S) * a.stage_bytes + 2 * kMaxStages * 8 +
                        4 * (G * kRPG * W + G * W * V + G);
    auto kern = k1_quantize_rows_staged_kernel<TPR, CPT, RP>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int grid = a.stages_total < sm_count() ? a.stages_total : sm_count();
    return launch_k(kern, dim3(grid), dim3(cons<TPR, RP>() + 32), smem, s, 1, a, status);
}

template <int CPT, int RP>
cudaError_t launch_staged_cpt(int nch, const __nv_bfloat16* X, const float* A, int M, int K, int r,
                              int8_t* Xq, float* sx, float* xA, int* status, cudaStream_t s) {
    constexpr int cap = staged::max_cons<RP>();
    const int need = (nch + CPT - 1) / CPT;  // threads per row
    if (need <= 32) return launch_staged<32, CPT, RP>(X, A, M, K, r, Xq, sx, xA, status, s);
    if (need <= 64) return launch_staged<64, CPT, RP>(X, A, M, K, r, Xq, sx, xA, status, s);
    if (need <= 96) return launch_staged<96, CPT, RP>(X, A, M, K, r, Xq, sx, xA, status, s);
    if (need <= 128) return launch_staged<128, CPT, RP>(X, A, M, K, r, Xq, sx, xA, status, s);
    if (need <= 192) return launch_staged<192, CPT, RP>(X, A, M, K, r, Xq, sx, xA, status, s);
    if (need <= 256) return launch_staged<256, CPT, RP>(X, A, M, K, r, Xq, sx, xA, status, s);
    if constexpr (cap >= 512) {
        if (need <= 384) return launch_staged<384, CPT, RP>(X, A, M, K, r, Xq, sx, xA, status, s);
        if (need <= 512) return launch_staged<512, CPT, RP>(X, A, M, K, r, Xq, sx, xA, status, s);
    }
    return cudaErrorNotSupported;
}

// one chunk per thread while a row fits the consumer threads, else two
template <int RP>
cudaError_t launch_staged_rp(const __nv_bfloat16* X, const float* A, int M, int K, int r,
                             int8_t* Xq, float* sx, float* xA, int* status, cudaStream_t s) {
    const int nch = K / 8;
    if (nch <= staged::max_cons<RP>())
        return launch_staged_cpt<1, RP>(nch, X, A, M, K, r, Xq, sx, xA, status, s);
    if constexpr (RP <= 4) {
        if (nch <= 2 * staged::max_cons<RP>())
            return launch_staged_cpt<2, RP>(nch, X, A, M, K, r, Xq, sx, xA, status, s);
    }
    return cudaErrorNotSupported;
}

// The staged kernel when it applies (bf16, r <= 8, at least 32M elements,
// rows short enough for the consumer threads at one or two chunks each);
// cudaErrorNotSupported otherwise.
cudaError_t launch_rows_staged(const __nv_bfloat16* X, const float* A, int M, int K, int r,
                               int8_t* Xq, float* sx, float* xA, int* status, cudaStream_t s) {
    // large inputs only: below ~64 MB of X the register-resident kernel
    // measured as fast or faster (the 1024 x 1024 MLP layers: slower here)
    if (static_cast<long long>(M) * K < (32LL << 20)) return cudaErrorNotSupported;
    if (r <= 4) return launch_staged_rp<4>(X, A, M, K, r, Xq, sx, xA, status, s);
    if (r <= 8) return launch_staged_rp<8>(X, A, M, K, r, Xq, sx, xA, status, s);
    return cudaErrorNotSupported;
}

template <typename T>
cudaError_t launch_rows_t(const T* X, const float* A, int M, int K, int r, int8_t* Xq, float* sx,
                          float* xA, cudaStream_t s) {
    if (r <= 4) return launch_rows_rp<T, 4>(X, A, M, K, r, Xq, sx, xA, s);
    if (r <= 8) return launch_rows_rp<T, 8>(X, A, M, K, r, Xq, sx, xA, s);
    if (r <= 16) return launch_rows_rp<T, 16>(X, A, M, K, r, Xq, sx, xA, s);
    return launch_rows_rp<T, 64>(X, A, M, K, r, Xq, sx, xA, s);
}

// ------------------------------------------------------------------ a0
// One CTA per 32 output channels.  Pass 1: column abs-max (coalesced rows of
// 32 floats).  Pass 2: 128 x 32 tiles transposed through shared memory so
// that Wq [N,K] rows are written contiguously.
constexpr int kQwCols = 32;
constexpr int kQwK = 128;

__global__ void __launch_bounds__(256) k_quantize_weight_kernel(const float* __restrict__ W, int K,
                                                                int N, int8_t* __restrict__ Wq,
                                                                float* __restrict__ sw) {
    __shared__ float part[8][kQwCols];
    __shared__ float inv_s[kQwCols];
    __shared__ float tile[kQwK][kQwCols + 1];
    const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;
    const int n0 = blockIdx.x * kQwCols;
    const int n = n0 + tx;
    float amax = 0.f;
    if (n < N)
        for (int k = ty; k < K; k += 8) amax = fmaxf(amax, fabsf(__ldg(W + static_cast<size_t>(k) * N + n)));
    part[ty][tx] = amax;
    __syncthreads();
    if (ty == 0) {
        float a = part[0][tx];
#pragma unroll
        for (int i = 1; i < 8; ++i) a = fmaxf(a, part[i][tx]);
        inv_s[tx] = a > 0.f ? __fdiv_rn(127.0f, a) : 0.f;
        if (n < N) sw[n] = __fdiv_rn(a, 127.0f);
    }
    __syncthreads();
    for (int k0 = 0; k0 < K; k0 += kQwK) {
        for (int kk = ty; kk < kQwK; kk += 8) {
            const int k = k0 + kk;
            tile[kk][tx] = (n < N && k < K) ? __ldg(W + static_cast<size_t>(k) * N + n) : 0.f;
        }
        __syncthreads();
        // 256 threads cover 32 channels x 8 groups of 16 consecutive k
        const int c = threadIdx.x / 8;
        const int g = threadIdx.x % 8;
        const int nn = n0 + c;
        if (nn < N) {
            const float inv = inv_s[c];
            int8_t* dst = Wq + static_cast<size_t>(nn) * K + k0 + g * 16;
            for (int e = 0; e < 16; ++e) {
                const int k = k0 + g * 16 + e;
                if (k < K) dst[e] = static_cast<int8_t>(quant_code(tile[g * 16 + e][c], inv));
            }
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_quantize_rows(Act act, const void* X, const float* A, int M, int K, int r,
                                 int8_t* Xq, float* sx, float* xA, int* status, cudaStream_t s) {
    if (act == kBF16) {
        const cudaError_t e = launch_rows_staged(static_cast<const __nv_bfloat16*>(X), A, M, K, r,
                                                 Xq, sx, xA, status, s);
        if (e != cudaErrorNotSupported) return e;
        return launch_rows_t(static_cast<const __nv_bfloat16*>(X), A, M, K, r, Xq, sx, xA, s);
    }
    return launch_rows_t(static_cast<const float*>(X), A, M, K, r, Xq, sx, xA, s);
}

cudaError_t launch_quantize_weight(const float* W, int K, int N, int8_t* Wq, float* sw,
                                   cudaStream_t s) {
    k_quantize_weight_kernel<<<(N + kQwCols - 1) / kQwCols, 256, 0, s>>>(W, K, N, Wq, sw);
    return cudaGetLastError();
}

}  // namespace qlora
