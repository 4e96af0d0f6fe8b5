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
// equation", for the shapes.)  This file holds the CUDA-core passes, used
// for fp32 activations (where the sums must stay fp32 throughout) and for dY
// rows that TMA cannot describe; bf16 layers run the tensor-core passes of
// k4_rank_tc.cu.  Each pass here streams its matrix once from HBM with
// 128-bit loads and does 2r FMAs per element.
//
// Layout of the work: a CTA owns 64 columns (8 lanes x 8, so a warp covers
// four rows per load) and a chunk of rows; the CL <= 8 CTAs that own the
// chunks of one column block form a thread-block cluster along the rows.
// Each CTA reduces its rows in registers and shared memory, then the cluster
// sums the CL partial results through distributed shared memory, rank by
// rank, so dB, dbias and dA leave the kernel final, with a fixed summation
// order (deterministic) and no second launch.  G's per-row sums over the
// column blocks stay as partial slices Gp in the workspace; the two
// consumers (the dX GEMM and the X pass) add the slices up themselves, or
// read G once launch_g_reduce has added many slices.
#include <cooperative_groups.h>

#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace qlora {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kLanesPerRow = 8;
constexpr int kCols = 8 * kLanesPerRow;             // 64 columns per CTA
constexpr int kRowsPerWarp = 32 / kLanesPerRow;     // 4 rows per warp-wide load
constexpr int kRowsPerPass = kRowsPerWarp * kWarps; // 32 rows per pass of the CTA
constexpr int kRJ = 8;                              // rank columns per sweep
constexpr int kMaxCluster = 8;
constexpr int kPassesInFlight = 4;
constexpr int kXRowBlock = 128;                     // rows whose G is staged at a time

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

// Sum of an 8-vector over the 8 lanes that share a row (xor offsets 4, 2, 1).
// On return, lane l holds the total of component l & 7.  Fixed order.
__device__ __forceinline__ float row_reduce8(float (&v)[8], int lane) {
    const bool b2 = lane & 4, b1 = lane & 2, b0 = lane & 1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b2 ? v[i] : v[i + 4];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 4);
        v[i] = (b2 ? v[i + 4] : v[i]) + recv;
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b1 ? v[i] : v[i + 2];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 2);
        v[i] = (b1 ? v[i + 2] : v[i]) + recv;
    }
    const float send = b0 ? v[0] : v[1];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
    return (b0 ? v[1] : v[0]) + recv;
}

// Sum over the four row groups of a warp (lanes with equal lane & 7).
__device__ __forceinline__ float warp_rows_sum(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    return v;
}

// Cluster sum of part[idx] over the CL ranks, rank 0 first, loads issued first.
__device__ __forceinline__ float cluster_sum(cg::cluster_group& cluster, float* part, int idx,
                                             int CL) {
    float v[kMaxCluster];
#pragma unroll
    for (int q = 0; q < kMaxCluster; ++q) v[q] = q < CL ? cluster.map_shared_rank(part, q)[idx] : 0.f;
    float s = v[0];
#pragma unroll
    for (int q = 1; q < kMaxCluster; ++q)
        if (q < CL) s += v[q];
    return s;
}

// ---------------------------------------------------------------- dY pass
template <typename T>
__global__ void __launch_bounds__(kThreads) k4_dy_kernel(
    const T* __restrict__ dY, const float* __restrict__ B, const float* __restrict__ xA, int M,
    int N, int r, int j0, int RM, float cscale, float* __restrict__ Gp, float* __restrict__ dB,
    float* __restrict__ dbias) {
    constexpr int kW = (kRJ + 1) * kCols;
    __shared__ float red[kWarps][kW];
    __shared__ float part[kW];
    pdl_trigger();
    pdl_wait();
    cg::cluster_group cluster = cg::this_cluster();
    const int CL = static_cast<int>(cluster.num_blocks());
    const int crank = static_cast<int>(cluster.block_rank());
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int rg = lane / kLanesPerRow, cl = lane % kLanesPerRow;
    const int cb = blockIdx.x;
    const int c0 = cb * kCols + cl * 8;
    const int mbeg = blockIdx.y * RM;
    const int mend = min(M, mbeg + RM);
    const bool vec = (N % 8) == 0;
    const int rowoff = warp * kRowsPerWarp + rg;

    float db[kRJ][8];
    float dbi[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        dbi[e] = 0.f;
#pragma unroll
        for (int j = 0; j < kRJ; ++j) db[j][e] = 0.f;
    }
    float bv[kRJ][8];
    bool have_b = false;

    for (int pb = mbeg; pb < mend; pb += kRowsPerPass * kPassesInFlight) {
        // every load of the pass group first: dY rows, their xA rows (and B once)
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
                xr[u][j] = (xA && ok && j0 + j < r) ? __ldg(xA + static_cast<size_t>(m) * r + j0 + j) : 0.f;
        }
        if (!have_b) {
#pragma unroll
            for (int j = 0; j < kRJ; ++j)
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    bv[j][e] = (B && j0 + j < r && c0 + e < N)
                                   ? __ldg(B + static_cast<size_t>(j0 + j) * N + c0 + e)
                                   : 0.f;
            have_b = true;
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
            const float gs = row_reduce8(g, lane);  // all lanes take part
            if (Gp && m < mend && j0 + cl < r) Gp[(static_cast<size_t>(cb) * M + m) * r + j0 + cl] = gs;
        }
    }

    // the four row groups of a warp, then the warps in order
#pragma unroll
    for (int j = 0; j < kRJ; ++j)
#pragma unroll
        for (int e = 0; e < 8; ++e) db[j][e] = warp_rows_sum(db[j][e]);
#pragma unroll
    for (int e = 0; e < 8; ++e) dbi[e] = warp_rows_sum(dbi[e]);
    if (rg == 0) {
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
        if (j < kRJ && (j0 + j >= r || dB == nullptr)) continue;
        if (j == kRJ && !with_bias) continue;
        const float s = cluster_sum(cluster, part, j * kCols + cc, CL);
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
    __shared__ __align__(16) float sG[kXRowBlock][kRJ];
    pdl_trigger();
    pdl_wait();
    cg::cluster_group cluster = cg::this_cluster();
    const int CL = static_cast<int>(cluster.num_blocks());
    const int crank = static_cast<int>(cluster.block_rank());
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int rg = lane / kLanesPerRow, cl = lane % kLanesPerRow;
    const int cb = blockIdx.x;
    const int c0 = cb * kCols + cl * 8;
    const int mbeg = blockIdx.y * RM;
    const int mend = min(M, mbeg + RM);
    const bool vec = (K % 8) == 0;
    const size_t gslice = static_cast<size_t>(M) * r;
    const int rowoff = warp * kRowsPerWarp + rg;

    float acc[8][kRJ];
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
        for (int j = 0; j < kRJ; ++j) acc[e][j] = 0.f;

    for (int rb = mbeg; rb < mend; rb += kXRowBlock) {
        const int rbe = min(mend, rb + kXRowBlock);
        // this block's X rows go out before G is staged
        float v[kXRowBlock / kRowsPerPass][8];
#pragma unroll
        for (int u = 0; u < kXRowBlock / kRowsPerPass; ++u) {
            const int m = rb + u * kRowsPerPass + rowoff;
            if (m < rbe) load8<T>(X + static_cast<size_t>(m) * K, c0, K, vec, v[u]);
            else
#pragma unroll
                for (int e = 0; e < 8; ++e) v[u][e] = 0.f;
        }
        __syncthreads();  // the previous block's G is no longer read
        for (int i = threadIdx.x; i < kXRowBlock * kRJ; i += kThreads) {
            const int rr = i / kRJ, j = i % kRJ;
            const int m = rb + rr;
            sG[rr][j] = (m < rbe && j0 + j < r)
                            ? sum_slices(Gp + static_cast<size_t>(m) * r + j0 + j, gslice, ncb)
                            : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kXRowBlock / kRowsPerPass; ++u) {
            const int rr = u * kRowsPerPass + rowoff;
            const float4 g0 = *reinterpret_cast<const float4*>(&sG[rr][0]);
            const float4 g1 = *reinterpret_cast<const float4*>(&sG[rr][4]);
            const float g[kRJ] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e)
#pragma unroll
                for (int j = 0; j < kRJ; ++j) acc[e][j] = fmaf(v[u][e], g[j], acc[e][j]);
        }
    }

#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
        for (int j = 0; j < kRJ; ++j) acc[e][j] = warp_rows_sum(acc[e][j]);
    if (rg == 0) {
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
        dA[static_cast<size_t>(k) * r + j0 + j] = cscale * cluster_sum(cluster, part, cc * kRJ + j, CL);
    }
    cluster.sync();
}

// G[m,j] = sum_b Gp[b][m,j] (only when a caller asks for G itself).
__global__ void k4_g_reduce_kernel(const float* __restrict__ Gp, int ncb, size_t n,
                                   float* __restrict__ G) {
    pdl_trigger();
    pdl_wait();
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
        G[i] = sum_slices(Gp + i, n, ncb);
}

// The same sums, four consecutive elements a thread (n % 4 == 0, 16-byte
// aligned slices) with sixteen slices' 16-byte loads in flight; each
// element's slices are still added in ascending order, so G is bit-identical.
__global__ void k4_g_reduce4_kernel(const float4* __restrict__ Gp, int ncb, size_t n4,
                                    float4* __restrict__ G) {
    pdl_trigger();
    pdl_wait();
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int b0 = 0; b0 < ncb; b0 += 16) {
            float4 v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
                if (b0 + u < ncb) v[u] = __ldg(Gp + static_cast<size_t>(b0 + u) * n4 + i);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                if (b0 + u >= ncb) break;
                if (b0 + u == 0) {
                    acc = v[u];
                } else {
                    acc.x += v[u].x;
                    acc.y += v[u].y;
                    acc.z += v[u].z;
                    acc.w += v[u].w;
                }
            }
        }
        G[i] = acc;
    }
}

// Cluster size along the rows.  The dY pass runs one CTA per SM (its
// accumulators fill the register file), so it takes clusters of at most 4:
// clusters of 8 such CTAs do not all fit in one wave of the GPCs.
int cluster_for(int M, int max_cl) {
    int cl = (M + 63) / 64;
    return cl > max_cl ? max_cl : (cl < 1 ? 1 : cl);
}

}  // namespace

bool rank_dy_tc(Act act, int N) { return act == kBF16 && N % 8 == 0; }

int rank_col_blocks(Act act, int N) {
    return rank_dy_tc(act, N) ? rank_tc_col_blocks(N) : (N + kCols - 1) / kCols;
}

cudaError_t launch_rank_dy(Act act, const void* dY, const float* B, const float* xA, int M, int N,
                           int r, float c, float* Gp, float* dB, float* dbias, int* status,
                           cudaStream_t s) {
    if (rank_dy_tc(act, N))
        return launch_rank_dy_tc(dY, B, xA, M, N, r, c, Gp, dB, dbias, status, s);
    const int cl = cluster_for(M, 4);
    const int RM = (M + cl - 1) / cl;
    const dim3 grid((N + kCols - 1) / kCols, cl);
    for (int j0 = 0; j0 < r; j0 += kRJ) {
        cudaError_t e;
        if (act == kBF16)
            e = launch_k(k4_dy_kernel<__nv_bfloat16>, grid, dim3(kThreads), 0, s, cl,
                         static_cast<const __nv_bfloat16*>(dY), B, xA, M, N, r, j0, RM, c, Gp, dB,
                         dbias);
        else
            e = launch_k(k4_dy_kernel<float>, grid, dim3(kThreads), 0, s, cl,
                         static_cast<const float*>(dY), B, xA, M, N, r, j0, RM, c, Gp, dB, dbias);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

cudaError_t launch_g_reduce(const float* Gp, int ncb, int M, int r, float* G, cudaStream_t s) {
    const size_t n = static_cast<size_t>(M) * r;
    if (n % 4 == 0 && (reinterpret_cast<uintptr_t>(Gp) & 15) == 0 && (reinterpret_cast<uintptr_t>(G) & 15) == 0) {
        const size_t n4 = n / 4;
        const int blocks = static_cast<int>((n4 + 127) / 128 < 2048 ? (n4 + 127) / 128 : 2048);
        return launch_k(k4_g_reduce4_kernel, dim3(blocks < 1 ? 1 : blocks), dim3(128), 0, s, 1,
                        reinterpret_cast<const float4*>(Gp), ncb, n4, reinterpret_cast<float4*>(G));
    }
    const int blocks = static_cast<int>((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
    return launch_k(k4_g_reduce_kernel, dim3(blocks < 1 ? 1 : blocks), dim3(256), 0, s, 1, Gp, ncb,
                    n, G);
}

cudaError_t launch_rank_x(Act act, const void* X, const float* G, int nsl, int M, int K, int r,
                          float c, float* dA, int* status, cudaStream_t s) {
    if (act == kBF16 && K % 8 == 0) return launch_rank_x_tc(X, G, nsl, M, K, r, c, dA, status, s);
    const int cl = cluster_for(M, kMaxCluster);
    const int RM = (M + cl - 1) / cl;
    const dim3 grid((K + kCols - 1) / kCols, cl);
    for (int j0 = 0; j0 < r; j0 += kRJ) {
        cudaError_t e;
        if (act == kBF16)
            e = launch_k(k4_x_kernel<__nv_bfloat16>, grid, dim3(kThreads), 0, s, cl,
                         static_cast<const __nv_bfloat16*>(X), G, nsl, M, K, r, j0, RM, c, dA);
        else
            e = launch_k(k4_x_kernel<float>, grid, dim3(kThreads), 0, s, cl,
                         static_cast<const float*>(X), G, nsl, M, K, r, j0, RM, c, dA);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace qlora
