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
// registers), writes M*K int8 codes, M scales and M*r floats of xA.
#include "internal.h"
#include "ptx.cuh"

namespace qlora {

namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 8;   // elements per 128-bit (bf16) / 2x128-bit (f32) load
constexpr int kMaxCPT = 8;  // chunks per thread held in registers
constexpr int kRJ = 8;      // xA columns accumulated per sweep

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

// Reduction over the TPR threads that share a row (TPR in {32,64,128,256}).
template <int TPR, bool IS_MAX>
__device__ __forceinline__ float row_reduce(float v, float* red, int row_in_block, int t) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        float w = __shfl_xor_sync(0xffffffffu, v, o);
        v = IS_MAX ? fmaxf(v, w) : v + w;
    }
    if constexpr (TPR > 32) {
        constexpr int W = TPR / 32;
        __syncwarp();
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

// One row per TPR threads; the row is read once into registers (K <= TPR*64).
template <typename T, int TPR>
__global__ void __launch_bounds__(kThreads) k1_quantize_rows_kernel(
    const T* __restrict__ X, const float* __restrict__ A, int M, int K, int r,
    int8_t* __restrict__ Xq, float* __restrict__ sx, float* __restrict__ xA) {
    constexpr int RPB = kThreads / TPR;
    __shared__ float red[RPB * (TPR / 32 > 0 ? TPR / 32 : 1)];
    const int row_in_block = threadIdx.x / TPR;
    const int t = threadIdx.x % TPR;
    const int m = blockIdx.x * RPB + row_in_block;
    const bool live = m < M;
    const int nchunks = K / kChunk;
    const T* xr = X + static_cast<size_t>(live ? m : 0) * K;

    float v[kMaxCPT][8];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxCPT; ++i) {
        const int ch = t + i * TPR;
        if (live && ch < nchunks) {
            Chunk8<T>::load(xr + ch * kChunk, v[i]);
#pragma unroll
            for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[i][e]));
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[i][e] = 0.f;
        }
    }
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

    // xA[m, j] = sum_k X[m,k] A[k,j], kRJ columns per sweep over the registers.
    for (int j0 = 0; j0 < r; j0 += kRJ) {
        float acc[kRJ];
#pragma unroll
        for (int j = 0; j < kRJ; ++j) acc[j] = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxCPT; ++i) {
            const int ch = t + i * TPR;
            if (live && ch < nchunks) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float* ar = A + static_cast<size_t>(ch * kChunk + e) * r + j0;
#pragma unroll
                    for (int j = 0; j < kRJ; ++j)
                        if (j0 + j < r) acc[j] = fmaf(v[i][e], __ldg(ar + j), acc[j]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kRJ; ++j) {
            float s = row_reduce<TPR, false>(acc[j], red, row_in_block, t);
            if (live && t == 0 && j0 + j < r) xA[static_cast<size_t>(m) * r + j0 + j] = s;
        }
    }
}

// Rows longer than 256*64 elements: two sweeps over global memory.
template <typename T>
__global__ void __launch_bounds__(kThreads) k1_quantize_rows_long_kernel(
    const T* __restrict__ X, const float* __restrict__ A, int M, int K, int r,
    int8_t* __restrict__ Xq, float* __restrict__ sx, float* __restrict__ xA) {
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
    for (int ch = t; ch < nchunks; ch += kThreads) {
        float v[8];
        Chunk8<T>::load(xr + ch * kChunk, v);
        *reinterpret_cast<uint2*>(qr + ch * kChunk) = pack8(v, inv);
    }
    if (t == 0) sx[m] = __fdiv_rn(amax, 127.0f);
    for (int j0 = 0; j0 < r; j0 += kRJ) {
        float acc[kRJ];
#pragma unroll
        for (int j = 0; j < kRJ; ++j) acc[j] = 0.f;
        for (int ch = t; ch < nchunks; ch += kThreads) {
            float v[8];
            Chunk8<T>::load(xr + ch * kChunk, v);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float* ar = A + static_cast<size_t>(ch * kChunk + e) * r + j0;
#pragma unroll
                for (int j = 0; j < kRJ; ++j)
                    if (j0 + j < r) acc[j] = fmaf(v[e], __ldg(ar + j), acc[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < kRJ; ++j) {
            float s = row_reduce<kThreads, false>(acc[j], red, 0, t);
            if (t == 0 && j0 + j < r) xA[static_cast<size_t>(m) * r + j0 + j] = s;
        }
    }
}

template <typename T>
cudaError_t launch_rows_t(const T* X, const float* A, int M, int K, int r, int8_t* Xq, float* sx,
                          float* xA, cudaStream_t s) {
    const int nchunks = K / kChunk;
    auto grid = [&](int tpr) { return dim3((M + kThreads / tpr - 1) / (kThreads / tpr)); };
    if (nchunks <= 32 * kMaxCPT)
        k1_quantize_rows_kernel<T, 32><<<grid(32), kThreads, 0, s>>>(X, A, M, K, r, Xq, sx, xA);
    else if (nchunks <= 64 * kMaxCPT)
        k1_quantize_rows_kernel<T, 64><<<grid(64), kThreads, 0, s>>>(X, A, M, K, r, Xq, sx, xA);
    else if (nchunks <= 128 * kMaxCPT)
        k1_quantize_rows_kernel<T, 128><<<grid(128), kThreads, 0, s>>>(X, A, M, K, r, Xq, sx, xA);
    else if (nchunks <= 256 * kMaxCPT)
        k1_quantize_rows_kernel<T, 256><<<grid(256), kThreads, 0, s>>>(X, A, M, K, r, Xq, sx, xA);
    else
        k1_quantize_rows_long_kernel<T><<<M, kThreads, 0, s>>>(X, A, M, K, r, Xq, sx, xA);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ a0
// One CTA per 32 output channels.  Pass 1: column abs-max (coalesced rows of
// 32 floats).  Pass 2: 32 x 128 tiles transposed through shared memory so that
// Wq [N,K] rows are written contiguously.
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
        // thread writes 4 consecutive k of one output channel: 8 channels x 32 threads...
        // 256 threads cover 32 channels x 8 groups of 16 k.
        const int c = threadIdx.x / 8;       // channel within the tile
        const int g = threadIdx.x % 8;       // 16 consecutive k per thread
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
                                 int8_t* Xq, float* sx, float* xA, cudaStream_t s) {
    if (act == kBF16)
        return launch_rows_t(static_cast<const __nv_bfloat16*>(X), A, M, K, r, Xq, sx, xA, s);
    return launch_rows_t(static_cast<const float*>(X), A, M, K, r, Xq, sx, xA, s);
}

cudaError_t launch_quantize_weight(const float* W, int K, int N, int8_t* Wq, float* sw,
                                   cudaStream_t s) {
    k_quantize_weight_kernel<<<(N + kQwCols - 1) / kQwCols, 256, 0, s>>>(W, K, N, Wq, sw);
    return cudaGetLastError();
}

}  // namespace qlora
