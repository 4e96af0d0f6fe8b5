// k4_rank.cu -- the skinny rank-r contractions of the LoRA backward:
//
//   Gp[b][m,j] = sum_{n in column block b} dY[m,n] B[j,n]   (G = sum_b Gp[b])
//   dB[j,n]    = c * sum_m xA[m,j] dY[m,n]                  (same pass over dY)
//   dbias[n]   = sum_m dY[m,n]                              (same pass over dY)
//   dA[k,j]    = c * sum_m X[m,k] G[m,j]                    (pass over X)
//
// ("How to fine-tune the 4-bit model?" thread: the LoRA factors are the
// trainable fp32 weights and the backward needs the A @ B.T-style adapter
// products; "Parameter-efficient fine-tuning of GPT-2 with LoRA", "LoRA
// equation", for the shapes.)  These are far too thin for tensor cores: each
// pass streams its matrix once from HBM with 128-bit loads and does 2r FMAs
// per element on CUDA cores.
//
// Layout of the work: a CTA owns 128 columns (16 lanes x 8) and a chunk of
// rows; the CL <= 8 CTAs that own the chunks of one column block form a
// thread-block cluster along the rows.  Each CTA reduces its rows in
// registers and shared memory, then the cluster sums the CL partial results
// through distributed shared memory, rank by rank, so dB, dbias and dA leave
// the kernel final, with a fixed summation order (deterministic) and no
// second launch.  G's per-row sums over the column blocks stay as partial
// slices Gp in the workspace; the two consumers (the dX GEMM and the X pass)
// add the slices up themselves.
#include <cooperative_groups.h>

#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace qlora {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCols = 128;         // columns per CTA: 16 lanes x 8
constexpr int kRJ = 8;             // rank columns per sweep
constexpr int kMaxCluster = 8;
constexpr int kRowsPerPass = 2 * kWarps;  // a half-warp per row
constexpr int kPassesInFlight = 4;
constexpr int kXRowBlock = 128;    // rows whose G is staged at a time (X pass)

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

// Sum of an 8-vector over the 16 lanes of a half-warp (xor offsets 8..1).  On
// return, lane l holds the total of component (l >> 1) & 7 when (l & 1) == 0.
__device__ __forceinline__ float half_reduce8(float (&v)[8], int lane) {
    const bool b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b3 ? v[i] : v[i + 4];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 8);
        v[i] = (b3 ? v[i + 4] : v[i]) + recv;
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b2 ? v[i] : v[i + 2];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 4);
        v[i] = (b2 ? v[i + 2] : v[i]) + recv;
    }
    {
        const float send = b1 ? v[0] : v[1];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 2);
        v[0] = (b1 ? v[1] : v[0]) + recv;
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// ---------------------------------------------------------------- dY pass
// Shared memory: red[kWarps][(kRJ + 1) * kCols] (per-warp partials) and
// part[(kRJ + 1) * kCols] (this CTA's partial, read by the cluster).
template <typename T>
__global__ void __launch_bounds__(kThreads) k4_dy_kernel(
    const T* __restrict__ dY, const float* __restrict__ B, const float* __restrict__ xA, int M,
    int N, int r, int j0, int RM, float cscale, float* __restrict__ Gp, float* __restrict__ dB,
    float* __restrict__ dbias) {
    constexpr int kW = (kRJ + 1) * kCols;
    __shared__ float red[kWarps][kW];
    __shared__ float part[kW];
    cg::cluster_group cluster = cg::this_cluster();
    const int CL = static_cast<int>(cluster.num_blocks());
    const int crank = static_cast<int>(cluster.block_rank());
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int half = lane >> 4, cl = lane & 15;
    const int cb = blockIdx.x;
    const int c0 = cb * kCols + cl * 8;
    const int mbeg = blockIdx.y * RM;
    const int mend = min(M, mbeg + RM);
    const bool vec = (N % 8) == 0;

    float bv[kRJ][8];
#pragma unroll
    for (int j = 0; j < kRJ; ++j)
#pragma unroll
        for (int e = 0; e < 8; ++e)
            bv[j][e] = (j0 + j < r && c0 + e < N) ? __ldg(B + static_cast<size_t>(j0 + j) * N + c0 + e) : 0.f;
    float db[kRJ][8];
    float dbi[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        dbi[e] = 0.f;
#pragma unroll
        for (int j = 0; j < kRJ; ++j) db[j][e] = 0.f;
    }

    const int rowoff = 2 * warp + half;
    for (int pb = mbeg; pb < mend; pb += kRowsPerPass * kPassesInFlight) {
        float v[kPassesInFlight][8];
        float xr[kPassesInFlight][kRJ];
#pragma unroll
        for (int u = 0; u < kPassesInFlight; ++u) {
            const int m = pb + u * kRowsPerPass + rowoff;
            const bool ok = m < mend;
            if (ok) load8<T>(dY + static_cast<size_t>(m) * N, c0, N, vec, v[u]);
            else
#pragma unroll
                for (int e = 0; e < 8; ++e) v[u][e] = 0.f;
#pragma unroll
            for (int j = 0; j < kRJ; ++j)
                xr[u][j] = (ok && j0 + j < r) ? __ldg(xA + static_cast<size_t>(m) * r + j0 + j) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kPassesInFlight; ++u) {
            const int m = pb + u * kRowsPerPass + rowoff;
            float g[kRJ];
#pragma unroll
            for (int j = 0; j < kRJ; ++j) {
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) s = fmaf(v[u][e], bv[j][e], s);
                g[j] = s;
#pragma unroll
                for (int e = 0; e < 8; ++e) db[j][e] = fmaf(xr[u][j], v[u][e], db[j][e]);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) dbi[e] += v[u][e];
            const float gs = half_reduce8(g, lane);  // all lanes take part
            const int jj = (cl >> 1) & 7;
            if (m < mend && (cl & 1) == 0 && j0 + jj < r)
                Gp[(static_cast<size_t>(cb) * M + m) * r + j0 + jj] = gs;
        }
    }

    // the two rows of a warp -> one partial per warp, then the warps in order
#pragma unroll
    for (int j = 0; j < kRJ; ++j)
#pragma unroll
        for (int e = 0; e < 8; ++e) db[j][e] += __shfl_xor_sync(0xffffffffu, db[j][e], 16);
#pragma unroll
    for (int e = 0; e < 8; ++e) dbi[e] += __shfl_xor_sync(0xffffffffu, dbi[e], 16);
    if (half == 0) {
#pragma unroll
        for (int j = 0; j < kRJ; ++j)
#pragma unroll
            for (int e = 0; e < 8; ++e) red[warp][j * kCols + cl * 8 + e] = db[j][e];
#pragma unroll
        for (int e = 0; e < 8; ++e) red[warp][kRJ * kCols + cl * 8 + e] = dbi[e];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kW; i += kThreads) {
        float s = red[0][i];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) s += red[w][i];
        part[i] = s;
    }
    cluster.sync();
    // rank q finalises its slice of the columns, summing the ranks in order
    const int per = (kCols + CL - 1) / CL;
    const int cbeg = crank * per;
    const int cend = min(kCols, cbeg + per);
    const bool with_bias = (j0 == 0) && dbias != nullptr;
    for (int i = threadIdx.x; i < (kRJ + 1) * (cend - cbeg); i += kThreads) {
        const int j = i / (cend - cbeg);
        const int cc = cbeg + i % (cend - cbeg);
        const int n = cb * kCols + cc;
        if (n >= N) continue;
        if (j < kRJ && j0 + j >= r) continue;
        if (j == kRJ && !with_bias) continue;
        float s = 0.f;
        for (int q = 0; q < CL; ++q) {
            const float* rp = cluster.map_shared_rank(part, q);
            s = q == 0 ? rp[j * kCols + cc] : s + rp[j * kCols + cc];
        }
        if (j < kRJ) dB[static_cast<size_t>(j0 + j) * N + n] = cscale * s;
        else dbias[n] = s;
    }
    cluster.sync();
}

// ---------------------------------------------------------------- X pass
// G for a block of rows is staged in shared memory from the Gp slices.
template <typename T>
__global__ void __launch_bounds__(kThreads) k4_x_kernel(
    const T* __restrict__ X, const float* __restrict__ Gp, int ncb, int M, int K, int r, int j0,
    int RM, float cscale, float* __restrict__ dA) {
    constexpr int kW = kCols * kRJ;
    __shared__ float red[kWarps][kW];
    __shared__ float part[kW];
    __shared__ float sG[kXRowBlock][kRJ];
    cg::cluster_group cluster = cg::this_cluster();
    const int CL = static_cast<int>(cluster.num_blocks());
    const int crank = static_cast<int>(cluster.block_rank());
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int half = lane >> 4, cl = lane & 15;
    const int cb = blockIdx.x;
    const int c0 = cb * kCols + cl * 8;
    const int mbeg = blockIdx.y * RM;
    const int mend = min(M, mbeg + RM);
    const bool vec = (K % 8) == 0;
    const size_t gslice = static_cast<size_t>(M) * r;

    float acc[8][kRJ];
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
        for (int j = 0; j < kRJ; ++j) acc[e][j] = 0.f;

    const int rowoff = 2 * warp + half;
    for (int rb = mbeg; rb < mend; rb += kXRowBlock) {
        const int rbe = min(mend, rb + kXRowBlock);
        __syncthreads();  // the previous block's G is no longer read
        for (int i = threadIdx.x; i < kXRowBlock * kRJ; i += kThreads) {
            const int rr = i / kRJ, j = i % kRJ;
            const int m = rb + rr;
            float s = 0.f;
            if (m < rbe && j0 + j < r) {
                const float* p = Gp + static_cast<size_t>(m) * r + j0 + j;
                s = __ldg(p);
                for (int b = 1; b < ncb; ++b) s += __ldg(p + b * gslice);
            }
            sG[rr][j] = s;
        }
        __syncthreads();
        for (int pb = rb; pb < rbe; pb += kRowsPerPass * kPassesInFlight) {
            float v[kPassesInFlight][8];
#pragma unroll
            for (int u = 0; u < kPassesInFlight; ++u) {
                const int m = pb + u * kRowsPerPass + rowoff;
                if (m < rbe) load8<T>(X + static_cast<size_t>(m) * K, c0, K, vec, v[u]);
                else
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[u][e] = 0.f;
            }
#pragma unroll
            for (int u = 0; u < kPassesInFlight; ++u) {
                const int rr = pb - rb + u * kRowsPerPass + rowoff;
                if (rr >= kXRowBlock) break;
                const float4 g0 = *reinterpret_cast<const float4*>(&sG[rr][0]);
                const float4 g1 = *reinterpret_cast<const float4*>(&sG[rr][4]);
                const float g[kRJ] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
                for (int e = 0; e < 8; ++e)
#pragma unroll
                    for (int j = 0; j < kRJ; ++j) acc[e][j] = fmaf(v[u][e], g[j], acc[e][j]);
            }
        }
    }

#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
        for (int j = 0; j < kRJ; ++j) acc[e][j] += __shfl_xor_sync(0xffffffffu, acc[e][j], 16);
    if (half == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
#pragma unroll
            for (int j = 0; j < kRJ; ++j) red[warp][(cl * 8 + e) * kRJ + j] = acc[e][j];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kW; i += kThreads) {
        float s = red[0][i];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) s += red[w][i];
        part[i] = s;
    }
    cluster.sync();
    const int per = (kCols + CL - 1) / CL;
    const int cbeg = crank * per;
    const int cend = min(kCols, cbeg + per);
    for (int i = threadIdx.x; i < (cend - cbeg) * kRJ; i += kThreads) {
        const int cc = cbeg + i / kRJ, j = i % kRJ;
        const int k = cb * kCols + cc;
        if (k >= K || j0 + j >= r) continue;
        float s = 0.f;
        for (int q = 0; q < CL; ++q) {
            const float* rp = cluster.map_shared_rank(part, q);
            s = q == 0 ? rp[cc * kRJ + j] : s + rp[cc * kRJ + j];
        }
        dA[static_cast<size_t>(k) * r + j0 + j] = cscale * s;
    }
    cluster.sync();
}

// G[m,j] = sum_b Gp[b][m,j] (only when a caller asks for G itself).
__global__ void k4_g_reduce_kernel(const float* __restrict__ Gp, int ncb, size_t n,
                                   float* __restrict__ G) {
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        float s = Gp[i];
        for (int b = 1; b < ncb; ++b) s += Gp[static_cast<size_t>(b) * n + i];
        G[i] = s;
    }
}

int cluster_for(int M) {
    int cl = (M + 63) / 64;
    return cl > kMaxCluster ? kMaxCluster : (cl < 1 ? 1 : cl);
}

template <typename Kern, typename... Args>
cudaError_t launch_clustered(Kern kern, dim3 grid, int cl, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = cl;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace

int rank_col_blocks(int N) { return (N + kCols - 1) / kCols; }

size_t rank_workspace_floats(int M, int N, int r) {
    return static_cast<size_t>(rank_col_blocks(N)) * M * r;
}

cudaError_t launch_rank_dy(Act act, const void* dY, const float* B, const float* xA, int M, int N,
                           int r, float c, float* Gp, float* dB, float* dbias, float* G,
                           cudaStream_t s) {
    const int cl = cluster_for(M);
    const int RM = (M + cl - 1) / cl;
    const dim3 grid(rank_col_blocks(N), cl);
    for (int j0 = 0; j0 < r; j0 += kRJ) {
        cudaError_t e;
        if (act == kBF16)
            e = launch_clustered(k4_dy_kernel<__nv_bfloat16>, grid, cl, s,
                                 static_cast<const __nv_bfloat16*>(dY), B, xA, M, N, r, j0, RM, c,
                                 Gp, dB, dbias);
        else
            e = launch_clustered(k4_dy_kernel<float>, grid, cl, s, static_cast<const float*>(dY), B,
                                 xA, M, N, r, j0, RM, c, Gp, dB, dbias);
        if (e != cudaSuccess) return e;
    }
    if (G) {
        const size_t n = static_cast<size_t>(M) * r;
        const int blocks = static_cast<int>((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
        k4_g_reduce_kernel<<<blocks, 256, 0, s>>>(Gp, rank_col_blocks(N), n, G);
    }
    return cudaGetLastError();
}

cudaError_t launch_rank_x(Act act, const void* X, const float* Gp, int ncb, int M, int K, int r,
                          float c, float* dA, cudaStream_t s) {
    const int cl = cluster_for(M);
    const int RM = (M + cl - 1) / cl;
    const dim3 grid(rank_col_blocks(K), cl);
    for (int j0 = 0; j0 < r; j0 += kRJ) {
        cudaError_t e;
        if (act == kBF16)
            e = launch_clustered(k4_x_kernel<__nv_bfloat16>, grid, cl, s,
                                 static_cast<const __nv_bfloat16*>(X), Gp, ncb, M, K, r, j0, RM, c, dA);
        else
            e = launch_clustered(k4_x_kernel<float>, grid, cl, s, static_cast<const float*>(X), Gp,
                                 ncb, M, K, r, j0, RM, c, dA);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace qlora
