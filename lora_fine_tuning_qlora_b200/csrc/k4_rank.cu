// k4_rank.cu -- the skinny rank-r contractions of the LoRA backward:
//
//   G[m,j]   = sum_n dY[m,n] B[j,n]          (pass over dY)
//   dB[j,n]  = c * sum_m xA[m,j] dY[m,n]     (same pass over dY)
//   dbias[n] = sum_m dY[m,n]                 (same pass over dY)
//   dA[k,j]  = c * sum_m X[m,k] G[m,j]       (pass over X)
//
// ("How to fine-tune the 4-bit model?" thread: the LoRA factors are the
// trainable fp32 weights and the backward needs the A @ B.T-style adapter
// products; "Parameter-efficient fine-tuning of GPT-2 with LoRA", "LoRA
// equation", for the shapes.)  These are far too thin for tensor cores: each
// pass streams its matrix once from HBM with 128-bit loads and does 2r FMAs
// per element on CUDA cores.
//
// Determinism: every sum has a fixed order.  A CTA owns a 256-column block
// and a chunk of rows; its lanes own 8 columns each and sweep the chunk's rows
// in a fixed order; per-row G partials are reduced inside the warp with a
// fixed butterfly, per-chunk dB/dbias/dA partials go to the workspace, and a
// second kernel sums the partials in chunk order.
#include "internal.h"
#include "ptx.cuh"

namespace qlora {

namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kCols = 256;  // columns per CTA: 32 lanes x 8
constexpr int kRJ = 8;      // rank columns per sweep

template <typename T>
__device__ __forceinline__ void load8(const T* row, int c0, int ncols, bool vec, float (&v)[8]) {
    if (vec && c0 + 8 <= ncols) {
        if constexpr (sizeof(T) == 2) {
            uint4 u = __ldg(reinterpret_cast<const uint4*>(row + c0));
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float2 f = __bfloat1622float2(h[i]);
                v[2 * i] = f.x;
                v[2 * i + 1] = f.y;
            }
        } else {
            float4 a = __ldg(reinterpret_cast<const float4*>(row + c0));
            float4 b = __ldg(reinterpret_cast<const float4*>(row + c0) + 1);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = (c0 + e < ncols) ? ActIO<T>::to_f(row[c0 + e]) : 0.f;
    }
}

// Sum of an 8-vector over the 32 lanes of a warp.  On return, lane l holds the
// total of component (l >> 2) & 7 when (l & 3) == 0.  Fixed order.
__device__ __forceinline__ float warp_reduce8(float (&v)[8], int lane) {
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b4 ? v[i] : v[i + 4];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
        v[i] = (b4 ? v[i + 4] : v[i]) + recv;
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b3 ? v[i] : v[i + 2];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 8);
        v[i] = (b3 ? v[i + 2] : v[i]) + recv;
    }
    {
        const float send = b2 ? v[0] : v[1];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 4);
        v[0] = (b2 ? v[1] : v[0]) + recv;
    }
    float s = v[0];
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    return s;
}

// Pass over dY for rank columns [j0, j0 + 8).
template <typename T>
__global__ void __launch_bounds__(kThreads) k4_dy_pass_kernel(
    const T* __restrict__ dY, const float* __restrict__ B, const float* __restrict__ xA, int M,
    int N, int r, int j0, int RM, float* __restrict__ Gp, float* __restrict__ dBp,
    float* __restrict__ dbp) {
    __shared__ float red[kWarps][kRJ + 1][kCols];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int cb = blockIdx.x, rc = blockIdx.y;
    const int c0 = cb * kCols + lane * 8;
    const int mbeg = rc * RM;
    const int mend = min(M, mbeg + RM);
    const bool vec = (N % 8) == 0;
    const bool with_bias = (j0 == 0) && dbp != nullptr;

    float bv[kRJ][8];
#pragma unroll
    for (int j = 0; j < kRJ; ++j)
#pragma unroll
        for (int e = 0; e < 8; ++e)
            bv[j][e] = (j0 + j < r && c0 + e < N) ? __ldg(B + static_cast<size_t>(j0 + j) * N + c0 + e) : 0.f;
    float db[kRJ][8];
    float dbias[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        dbias[e] = 0.f;
#pragma unroll
        for (int j = 0; j < kRJ; ++j) db[j][e] = 0.f;
    }

    for (int m = mbeg + warp; m < mend; m += kWarps) {
        float v[8];
        load8<T>(dY + static_cast<size_t>(m) * N, c0, N, vec, v);
        float xa[kRJ];
#pragma unroll
        for (int j = 0; j < kRJ; ++j) xa[j] = (j0 + j < r) ? __ldg(xA + static_cast<size_t>(m) * r + j0 + j) : 0.f;
        float g[kRJ];
#pragma unroll
        for (int j = 0; j < kRJ; ++j) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) s = fmaf(v[e], bv[j][e], s);
            g[j] = s;
#pragma unroll
            for (int e = 0; e < 8; ++e) db[j][e] = fmaf(xa[j], v[e], db[j][e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) dbias[e] += v[e];
        const float gs = warp_reduce8(g, lane);
        const int jj = (lane >> 2) & 7;
        if ((lane & 3) == 0 && j0 + jj < r)
            Gp[(static_cast<size_t>(cb) * M + m) * r + j0 + jj] = gs;
    }

    // combine the warps of this CTA (fixed order), write the chunk's partials
#pragma unroll
    for (int j = 0; j < kRJ; ++j)
#pragma unroll
        for (int e = 0; e < 8; ++e) red[warp][j][lane * 8 + e] = db[j][e];
#pragma unroll
    for (int e = 0; e < 8; ++e) red[warp][kRJ][lane * 8 + e] = dbias[e];
    __syncthreads();
    for (int i = threadIdx.x; i < (kRJ + 1) * kCols; i += kThreads) {
        const int j = i / kCols, cl = i % kCols;
        const int n = cb * kCols + cl;
        if (n >= N) continue;
        float s = red[0][j][cl];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) s += red[w][j][cl];
        if (j < kRJ) {
            if (j0 + j < r) dBp[(static_cast<size_t>(rc) * r + j0 + j) * N + n] = s;
        } else if (with_bias) {
            dbp[static_cast<size_t>(rc) * N + n] = s;
        }
    }
}

// Pass over X for rank columns [j0, j0 + 8): dA partials [chunk][K][r].
template <typename T>
__global__ void __launch_bounds__(kThreads) k4_x_pass_kernel(const T* __restrict__ X,
                                                             const float* __restrict__ G, int M,
                                                             int K, int r, int j0, int RM,
                                                             float* __restrict__ dAp) {
    __shared__ float red[kWarps][kCols][kRJ + 1];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int cb = blockIdx.x, rc = blockIdx.y;
    const int c0 = cb * kCols + lane * 8;
    const int mbeg = rc * RM;
    const int mend = min(M, mbeg + RM);
    const bool vec = (K % 8) == 0;
    float acc[8][kRJ];
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
        for (int j = 0; j < kRJ; ++j) acc[e][j] = 0.f;
    for (int m = mbeg + warp; m < mend; m += kWarps) {
        float v[8];
        load8<T>(X + static_cast<size_t>(m) * K, c0, K, vec, v);
        float g[kRJ];
#pragma unroll
        for (int j = 0; j < kRJ; ++j) g[j] = (j0 + j < r) ? __ldg(G + static_cast<size_t>(m) * r + j0 + j) : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e)
#pragma unroll
            for (int j = 0; j < kRJ; ++j) acc[e][j] = fmaf(v[e], g[j], acc[e][j]);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
        for (int j = 0; j < kRJ; ++j) red[warp][lane * 8 + e][j] = acc[e][j];
    __syncthreads();
    for (int i = threadIdx.x; i < kCols * kRJ; i += kThreads) {
        const int cl = i / kRJ, j = i % kRJ;
        const int k = cb * kCols + cl;
        if (k >= K || j0 + j >= r) continue;
        float s = red[0][cl][j];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) s += red[w][cl][j];
        dAp[(static_cast<size_t>(rc) * K + k) * r + j0 + j] = s;
    }
}

// G = sum over column blocks, dB = c * sum over row chunks, dbias likewise.
__global__ void k4_reduce_dy_kernel(const float* __restrict__ Gp, const float* __restrict__ dBp,
                                    const float* __restrict__ dbp, int M, int N, int r, int ncb,
                                    int nrc, float c, float* __restrict__ G, float* __restrict__ dB,
                                    float* __restrict__ dbias) {
    const size_t nG = static_cast<size_t>(M) * r;
    const size_t nB = static_cast<size_t>(r) * N;
    const size_t nb = dbias ? static_cast<size_t>(N) : 0;
    const size_t total = nG + nB + nb;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        if (i < nG) {
            float s = Gp[i];
            for (int b = 1; b < ncb; ++b) s += Gp[static_cast<size_t>(b) * nG + i];
            G[i] = s;
        } else if (i < nG + nB) {
            const size_t o = i - nG;
            float s = dBp[o];
            for (int b = 1; b < nrc; ++b) s += dBp[static_cast<size_t>(b) * nB + o];
            dB[o] = c * s;
        } else {
            const size_t o = i - nG - nB;
            float s = dbp[o];
            for (int b = 1; b < nrc; ++b) s += dbp[static_cast<size_t>(b) * N + o];
            dbias[o] = s;
        }
    }
}

__global__ void k4_reduce_x_kernel(const float* __restrict__ dAp, int K, int r, int nrc, float c,
                                   float* __restrict__ dA) {
    const size_t n = static_cast<size_t>(K) * r;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        float s = dAp[i];
        for (int b = 1; b < nrc; ++b) s += dAp[static_cast<size_t>(b) * n + i];
        dA[i] = c * s;
    }
}

int chunks_for(int M, int col_blocks) {
    // about two CTAs per SM, at least 8 rows per chunk
    int want = (2 * 148 + col_blocks - 1) / col_blocks;
    int maxc = (M + 7) / 8;
    if (want > maxc) want = maxc;
    if (want < 1) want = 1;
    return want;
}

}  // namespace

RankPlan plan_rank(int M, int K, int N, int r) {
    (void)r;
    RankPlan p;
    p.n_col_blocks = (N + kCols - 1) / kCols;
    int nc = chunks_for(M, p.n_col_blocks);
    p.rows_per_chunk = (M + nc - 1) / nc;
    p.n_chunks = (M + p.rows_per_chunk - 1) / p.rows_per_chunk;
    const int kcb = (K + kCols - 1) / kCols;
    int kc = chunks_for(M, kcb);
    p.rows_per_kchunk = (M + kc - 1) / kc;
    p.k_chunks = (M + p.rows_per_kchunk - 1) / p.rows_per_kchunk;
    return p;
}

size_t rank_workspace_floats(const RankPlan& p, int M, int K, int N, int r) {
    const size_t gp = static_cast<size_t>(p.n_col_blocks) * M * r;
    const size_t dbp = static_cast<size_t>(p.n_chunks) * r * N;
    const size_t dbias = static_cast<size_t>(p.n_chunks) * N;
    const size_t dap = static_cast<size_t>(p.k_chunks) * K * r;
    // the dY-pass partials and the X-pass partials are live at different times
    const size_t dy = gp + dbp + dbias;
    return dy > dap ? dy : dap;
}

cudaError_t launch_rank_dy(Act act, const void* dY, const float* B, const float* xA, int M, int N,
                           int r, float c, const RankPlan& p, float* G, float* dB, float* dbias,
                           float* wsf, cudaStream_t s) {
    float* Gp = wsf;
    float* dBp = Gp + static_cast<size_t>(p.n_col_blocks) * M * r;
    float* dbp = dBp + static_cast<size_t>(p.n_chunks) * r * N;
    dim3 grid(p.n_col_blocks, p.n_chunks);
    for (int j0 = 0; j0 < r; j0 += kRJ) {
        if (act == kBF16)
            k4_dy_pass_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(
                static_cast<const __nv_bfloat16*>(dY), B, xA, M, N, r, j0, p.rows_per_chunk, Gp,
                dBp, dbias ? dbp : nullptr);
        else
            k4_dy_pass_kernel<float><<<grid, kThreads, 0, s>>>(static_cast<const float*>(dY), B, xA,
                                                               M, N, r, j0, p.rows_per_chunk, Gp,
                                                               dBp, dbias ? dbp : nullptr);
    }
    const size_t total = static_cast<size_t>(M) * r + static_cast<size_t>(r) * N + (dbias ? N : 0);
    int blocks = static_cast<int>((total + 255) / 256);
    if (blocks > 4 * 148) blocks = 4 * 148;
    k4_reduce_dy_kernel<<<blocks, 256, 0, s>>>(Gp, dBp, dbp, M, N, r, p.n_col_blocks, p.n_chunks, c,
                                                G, dB, dbias);
    return cudaGetLastError();
}

cudaError_t launch_rank_x(Act act, const void* X, const float* G, int M, int K, int r, float c,
                          const RankPlan& p, float* dA, float* wsf, cudaStream_t s) {
    float* dAp = wsf;
    dim3 grid((K + kCols - 1) / kCols, p.k_chunks);
    for (int j0 = 0; j0 < r; j0 += kRJ) {
        if (act == kBF16)
            k4_x_pass_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(
                static_cast<const __nv_bfloat16*>(X), G, M, K, r, j0, p.rows_per_kchunk, dAp);
        else
            k4_x_pass_kernel<float><<<grid, kThreads, 0, s>>>(static_cast<const float*>(X), G, M, K,
                                                              r, j0, p.rows_per_kchunk, dAp);
    }
    const size_t total = static_cast<size_t>(K) * r;
    int blocks = static_cast<int>((total + 255) / 256);
    if (blocks > 4 * 148) blocks = 4 * 148;
    k4_reduce_x_kernel<<<blocks, 256, 0, s>>>(dAp, K, r, p.k_chunks, c, dA);
    return cudaGetLastError();
}

}  // namespace qlora
