// outlier.cu -- the one-off quantization of an outlier-compensated int8
// kernel (keras-llm-light, "Weights quantization" and "Simplified
// Int8Variable quantization": the weights are quantized after removing
// outliers at a 99.9 percentile cutoff, the outliers are kept in fp16 in a
// sparse list, and the kernel is rebuilt as bias + value * scale with the
// outliers written back; the block summary stores such kernels as uint8).
//
// Readings (the pages give no formula): one affine code per tensor; lo and hi
// are the 0.1th and 99.9th percentiles of all K*N entries (linear
// interpolation between the order statistics at (n - 1) p / 100, in fp64,
// stored as fp32); entries strictly outside [lo, hi] are outliers, kept as
// fp16 (round to nearest even) with code 0; scale = fl32((hi - lo) / 255),
// bias = lo, and every other entry gets
// code = clamp(rne(fl32(fl32(w - bias) / scale)), 0, 255) (0 when scale is 0).
//
// On the GPU: the four order statistics are found by a radix select (four
// 8-bit digit rounds over order-preserving integer keys; a grid-wide
// histogram pass and a one-block digit choice per round), the cutoffs and the
// affine parameters by one thread in fp64, the codes by a tiled pass that
// writes both layouts ([N,K] for the dX GEMM, [K,N] for the forward GEMM)
// and counts the outliers of every (row, 128-column block) bucket, then a
// one-block exclusive scan gives the bucket starts and a last pass scatters
// the outliers into their buckets.  The order inside a bucket is not fixed;
// the set is.
#include "internal.h"
#include "ptx.cuh"

#include <cuda_fp16.h>
#include <math.h>

namespace qlora {

namespace {

constexpr int kTargets = 4;   // order statistics: s[i_lo], s[i_lo + 1], s[i_hi], s[i_hi + 1]
constexpr int kBins = 256;

__device__ __forceinline__ uint32_t f2key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key2f(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

struct SelState {
    uint32_t prefix[kTargets];  // digits decided so far (high bits)
    uint32_t rank[kTargets];    // rank within the elements matching the prefix
};

__global__ void __launch_bounds__(256) ol_hist_kernel(const float* __restrict__ W, long n, int round,
                                                      const SelState* __restrict__ st,
                                                      unsigned int* __restrict__ hist) {
    __shared__ unsigned int h[kTargets][kBins];
    for (int i = threadIdx.x; i < kTargets * kBins; i += blockDim.x) (&h[0][0])[i] = 0u;
    __syncthreads();
    const int shift = 24 - 8 * round;
    const uint32_t hi_mask = round == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
    uint32_t pre[kTargets];
#pragma unroll
    for (int t = 0; t < kTargets; ++t) pre[t] = st->prefix[t] & hi_mask;
    for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long>(gridDim.x) * blockDim.x) {
        const uint32_t k = f2key(__ldg(W + i));
        const uint32_t d = (k >> shift) & 0xFFu;
#pragma unroll
        for (int t = 0; t < kTargets; ++t)
            if ((k & hi_mask) == pre[t]) atomicAdd(&h[t][d], 1u);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kTargets * kBins; i += blockDim.x) {
        const unsigned int v = (&h[0][0])[i];
        if (v) atomicAdd(hist + i, v);
    }
}

// One block of kTargets warps: warp t picks the digit of target t for this
// round and clears its histogram for the next.
__global__ void __launch_bounds__(32 * kTargets) ol_select_kernel(int round, SelState* st,
                                                                   unsigned int* hist) {
    const int t = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int shift = 24 - 8 * round;
    unsigned int* h = hist + t * kBins;
    // counts of the lane's 8 bins, then a warp prefix over the lanes
    unsigned int c[8], sum = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
        c[b] = h[lane * 8 + b];
        sum += c[b];
    }
    unsigned int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    const unsigned int excl = incl - sum;
    const unsigned int rank = st->rank[t];
    const bool mine = rank >= excl && rank < incl;
    unsigned int digit = 0, below = 0;
    if (mine) {
        unsigned int acc = excl;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            if (rank >= acc && rank < acc + c[b]) {
                digit = lane * 8 + b;
                below = acc;
            }
            acc += c[b];
        }
    }
    const unsigned int who = __ballot_sync(0xffffffffu, mine);
    const int src = who ? __ffs(who) - 1 : 0;
    digit = __shfl_sync(0xffffffffu, digit, src);
    below = __shfl_sync(0xffffffffu, below, src);
    __syncwarp();
    if (lane == 0) {
        st->prefix[t] |= digit << shift;
        st->rank[t] = rank - below;
    }
#pragma unroll
    for (int b = 0; b < 8; ++b) h[lane * 8 + b] = 0u;
}

// i = floor((n - 1) p / 100) for p = 0.1 and 99.9, exactly as the host does.
__device__ __forceinline__ void pct_pos(long n, double p, long* i, double* frac) {
    const double h = static_cast<double>(n - 1) * p / 100.0;
    long ii = static_cast<long>(floor(h));
    if (ii >= n - 1) ii = n - 1;
    *i = ii;
    *frac = h - static_cast<double>(ii);
}

__global__ void ol_init_kernel(long n, SelState* st) {
    long i0, i1;
    double f;
    pct_pos(n, 0.1, &i0, &f);
    pct_pos(n, 99.9, &i1, &f);
    const long t[kTargets] = {i0, i0 + 1 < n ? i0 + 1 : i0, i1, i1 + 1 < n ? i1 + 1 : i1};
    for (int k = 0; k < kTargets; ++k) {
        st->prefix[k] = 0u;
        st->rank[k] = static_cast<uint32_t>(t[k]);
    }
}

// lo, hi by linear interpolation in fp64; scale and bias in fp32.
__global__ void ol_params_kernel(long n, const SelState* st, float* par) {
    float v[kTargets];
    for (int k = 0; k < kTargets; ++k) v[k] = key2f(st->prefix[k]);
    long i;
    double f;
    pct_pos(n, 0.1, &i, &f);
    double q = static_cast<double>(v[0]);
    if (i + 1 < n && f > 0.0) q += f * (static_cast<double>(v[1]) - static_cast<double>(v[0]));
    const float lo = static_cast<float>(q);
    pct_pos(n, 99.9, &i, &f);
    q = static_cast<double>(v[2]);
    if (i + 1 < n && f > 0.0) q += f * (static_cast<double>(v[3]) - static_cast<double>(v[2]));
    const float hi = static_cast<float>(q);
    par[0] = lo;
    par[1] = hi;
    par[2] = __fdiv_rn(__fsub_rn(hi, lo), 255.0f);
    par[3] = lo;
}

__device__ __forceinline__ uint8_t affine_code(float w, float scale, float bias) {
    if (!(scale > 0.f)) return 0;
    float r = rintf(__fdiv_rn(__fsub_rn(w, bias), scale));
    r = r < 0.f ? 0.f : (r > 255.f ? 255.f : r);
    return static_cast<uint8_t>(r);
}

// 32 x 32 tiles of W [K,N]: codes in both layouts; outliers counted per
// (row, 128-column block) bucket of each layout.
constexpr int kT = 32;

__global__ void __launch_bounds__(256) ol_codes_kernel(const float* __restrict__ W, int K, int N,
                                                       const float* __restrict__ par,
                                                       uint8_t* __restrict__ codes_nk,
                                                       uint8_t* __restrict__ codes_kn,
                                                       int* __restrict__ cnt_nk, int* __restrict__ cnt_kn) {
    __shared__ uint8_t tile[kT][kT + 4];
    const float lo = par[0], hi = par[1], scale = par[2], bias = par[3];
    const int k0 = blockIdx.y * kT, n0 = blockIdx.x * kT;
    const int tx = threadIdx.x % kT, ty = threadIdx.x / kT;  // 32 x 8
    const int nbK = (K + 127) / 128, nbN = (N + 127) / 128;
    for (int kk = ty; kk < kT; kk += 8) {
        const int k = k0 + kk, n = n0 + tx;
        uint8_t code = 0;
        if (k < K && n < N) {
            const float w = __ldg(W + static_cast<size_t>(k) * N + n);
            if (w < lo || w > hi) {
                atomicAdd(cnt_nk + static_cast<size_t>(n) * nbK + k / 128, 1);
                atomicAdd(cnt_kn + static_cast<size_t>(k) * nbN + n / 128, 1);
            } else {
                code = affine_code(w, scale, bias);
            }
            codes_kn[static_cast<size_t>(k) * N + n] = code;
        }
        tile[kk][tx] = code;
    }
    __syncthreads();
    for (int nn = ty; nn < kT; nn += 8) {
        const int n = n0 + nn, k = k0 + tx;
        if (n < N && k < K) codes_nk[static_cast<size_t>(n) * K + k] = tile[tx][nn];
    }
}

// Exclusive scan of cnt [S] into start [S + 1] by one block; cnt is cleared
// (it is the scatter's fill counter next).
__global__ void __launch_bounds__(1024) ol_scan_kernel(int* __restrict__ cnt, int* __restrict__ start,
                                                       long S) {
    __shared__ int part[1024];
    const int t = threadIdx.x;
    const long per = (S + 1023) / 1024;
    const long b = t * per, e = b + per < S ? b + per : S;
    int sum = 0;
    for (long i = b; i < e; ++i) sum += cnt[i];
    part[t] = sum;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        const int v = t >= o ? part[t - o] : 0;
        __syncthreads();
        part[t] += v;
        __syncthreads();
    }
    int run = part[t] - sum;
    for (long i = b; i < e; ++i) {
        start[i] = run;
        run += cnt[i];
        cnt[i] = 0;
    }
    if (t == 1023) start[S] = part[1023];
}

__global__ void __launch_bounds__(256) ol_scatter_kernel(const float* __restrict__ W, int K, int N,
                                                         const float* __restrict__ par,
                                                         const int* __restrict__ start_nk,
                                                         int* __restrict__ fill_nk,
                                                         uint32_t* __restrict__ ent_nk,
                                                         const int* __restrict__ start_kn,
                                                         int* __restrict__ fill_kn,
                                                         uint32_t* __restrict__ ent_kn, int cap) {
    const float lo = par[0], hi = par[1];
    const int nbK = (K + 127) / 128, nbN = (N + 127) / 128;
    const long total = static_cast<long>(K) * N;
    for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long>(gridDim.x) * blockDim.x) {
        const float w = __ldg(W + i);
        if (!(w < lo || w > hi)) continue;
        const int k = static_cast<int>(i / N), n = static_cast<int>(i % N);
        const uint32_t h = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(w)));
        const size_t bnk = static_cast<size_t>(n) * nbK + k / 128;
        const int pnk = start_nk[bnk] + atomicAdd(fill_nk + bnk, 1);
        if (pnk < cap) ent_nk[pnk] = (static_cast<uint32_t>(k % 128) << 16) | h;
        const size_t bkn = static_cast<size_t>(k) * nbN + n / 128;
        const int pkn = start_kn[bkn] + atomicAdd(fill_kn + bkn, 1);
        if (pkn < cap) ent_kn[pkn] = (static_cast<uint32_t>(n % 128) << 16) | h;
    }
}

}  // namespace

size_t outlier_buckets_nk(int K, int N) { return static_cast<size_t>(N) * ((K + 127) / 128); }
size_t outlier_buckets_kn(int K, int N) { return static_cast<size_t>(K) * ((N + 127) / 128); }

size_t outlier_workspace_bytes(int K, int N) {
    const size_t a = 1024 + sizeof(SelState) + kTargets * kBins * 4;
    return ((a + 255) & ~size_t(255)) + 4 * (outlier_buckets_nk(K, N) + outlier_buckets_kn(K, N)) + 256;
}

cudaError_t launch_quantize_outlier(const float* W, int K, int N, const OutlierKernel& q,
                                    void* workspace, cudaStream_t s) {
    const long n = static_cast<long>(K) * N;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    SelState* st = reinterpret_cast<SelState*>(ws);
    unsigned int* hist = reinterpret_cast<unsigned int*>(ws + 1024);
    const size_t a = 1024 + sizeof(SelState) + kTargets * kBins * 4;
    int* cnt_nk = reinterpret_cast<int*>(ws + ((a + 255) & ~size_t(255)));
    int* cnt_kn = cnt_nk + outlier_buckets_nk(K, N);
    cudaError_t e = cudaMemsetAsync(hist, 0, kTargets * kBins * 4, s);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(cnt_nk, 0, 4 * (outlier_buckets_nk(K, N) + outlier_buckets_kn(K, N)), s);
    if (e != cudaSuccess) return e;
    ol_init_kernel<<<1, 1, 0, s>>>(n, st);
    const int hb = static_cast<int>(n / 256 / 8 + 1 < 4 * sm_count() ? n / 256 / 8 + 1 : 4 * sm_count());
    for (int round = 0; round < 4; ++round) {
        ol_hist_kernel<<<hb, 256, 0, s>>>(W, n, round, st, hist);
        ol_select_kernel<<<1, 32 * kTargets, 0, s>>>(round, st, hist);
    }
    ol_params_kernel<<<1, 1, 0, s>>>(n, st, q.par);
    const dim3 cg((N + kT - 1) / kT, (K + kT - 1) / kT);
    ol_codes_kernel<<<cg, 256, 0, s>>>(W, K, N, q.par, q.codes_nk, q.codes_kn, cnt_nk, cnt_kn);
    ol_scan_kernel<<<1, 1024, 0, s>>>(cnt_nk, q.start_nk, static_cast<long>(outlier_buckets_nk(K, N)));
    ol_scan_kernel<<<1, 1024, 0, s>>>(cnt_kn, q.start_kn, static_cast<long>(outlier_buckets_kn(K, N)));
    ol_scatter_kernel<<<hb, 256, 0, s>>>(W, K, N, q.par, q.start_nk, cnt_nk, q.ent_nk, q.start_kn, cnt_kn,
                                         q.ent_kn, q.cap);
    return cudaGetLastError();
}

}  // namespace qlora
