// small_m.cu -- the two GEMMs of the layer for few tokens (M <= 64), where
// the int8 kernel Wq [N,K] dominates the traffic and every SM must stream a
// share of it ("How to fine-tune the 4-bit model?" thread: with few tokens
// the layer is bound by reading the weights, not by arithmetic).
//
// Tokens go on the MMA's N (16 .. 64, padded to 16) and 128 output channels
// on its M, so one CTA's accumulator holds all tokens of its channels; the
// contraction is split over a cluster of S CTAs (along y) so that
// ceil(channels / 128) x S CTAs cover the SMs:
//
//   forward  acc^T[n, m] = sum_k Wq[n,k] Xq[m,k]            tcgen05 kind::i8
//            Y[m,n] = acc sx[m] sw[n] + bias[n] + c sum_j xA[m,j] B[j,n]
//   dX       dX^T[k, m] = sum_n (Wq[n,k] sw[n]) dY[m,n]      tcgen05 kind::f16
//            dX[m,k] += c sum_j G[m,j] A[k,j]   (then the ReLU gate, if any)
//
// The forward's operands arrive by TMA (Wq as a 128 x 128 K-major tile, Xq
// as MP x 128, both with the 128-byte swizzle); the dX kernel's Wq codes are
// read by eight de-quantize warps into an MN-major bf16 tile (128 channels x
// 64 contraction rows, the layout of the large dX kernels' B operand, here
// the A operand), dY arrives by TMA (MP x 64, K-major).
//
// Reduction over the split: after every CTA's accumulator is final (cluster
// barrier), each CTA stores its partial sums of token columns [q W, q W + W)
// (W = MP / S) into the shared memory of CTA q (distributed shared memory,
// into the now idle operand ring), a second cluster barrier publishes them,
// and CTA q adds the S partials in rank order (exact for int32, a fixed
// order for fp32) and writes its columns.  Every wait is bounded.
#include "internal.h"
#include "ptx.cuh"
#include "dx_common.cuh"

namespace qlora {

namespace {

constexpr int kCh = 128;                 // output channels per CTA (the MMA's M)
constexpr int kRing = 192 * 1024;        // operand ring; later the partial-sum buffer
constexpr int kTabFloats = 256 * 17;     // per owner column: the row's rank-r factor row and scale
constexpr int kBarOff = kRing + kTabFloats * 4;  // barriers after the ring and the table
constexpr int kMaxStages = 8;
constexpr int kEpiW = 4;                 // epilogue warps: one per TMEM lane quarter
constexpr int kDqW = 8;                  // de-quantize warps (dX)
constexpr int kFwdThreads = 32 * (2 + kEpiW);
constexpr int kDxThreads = 32 * (2 + kDqW + kEpiW);
constexpr int kMaxSplit = 8;
constexpr int kMaxTokens = 64;           // above this the large-tile kernels measured as fast or faster

struct SmallArgs {
    int M, N, K;          // the layer's shapes (tokens, out_features, in_features)
    int MP;               // tokens padded to a multiple of 16
    int S;                // split of the contraction (cluster size along y)
    int stages;           // ring depth
    int kblocks;          // contraction blocks in total
    uint32_t tmem_cols;
};

__device__ __forceinline__ void cluster_sync_all() {
    cluster_arrive();
    cluster_wait();
}

// smem: [ring kRing][barriers]
__device__ __forceinline__ uint8_t* aligned_smem(uint8_t* raw) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~static_cast<uintptr_t>(1023));
}

// Sends this CTA's partial accumulator (TMEM lanes = channels, columns =
// tokens) to the owners of its token columns: recv[source rank][column][row]
// at the owner, the 32 rows of a warp in consecutive words (no bank
// conflicts).  Warp q of the epilogue holds lane quarter q.
__device__ __forceinline__ void send_partials(uint32_t tmem, int q, int lane, int MP, int W, uint32_t rank,
                                              const uint32_t* recv_local) {
    const uint32_t base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int row = q * 32 + lane;
    for (int c0 = 0; c0 < MP; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(base + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int c = c0 + e;
            const int owner = c / W;
            const uint32_t off = (static_cast<uint32_t>(rank) * W + (c - owner * W)) * kCh + row;
            dsmem_st(dsmem_addr(recv_local + off, static_cast<uint32_t>(owner)), __uint_as_float(v[e]));
        }
    }
}

// ------------------------------------------------------------------ forward
// W4: the kernel is packed int4 codes Wp [N, K/2]; TMA brings each stage's
// packed tile ([128 rows][64 bytes], no swizzle) and the epilogue warps,
// idle until the accumulator is final, expand it into the int8 tile in the
// layout the TMA would have written (16-byte chunk c of row n at c ^ (n % 8)).
template <typename OutT, int RMAX, bool W4>
__global__ void __launch_bounds__(kFwdThreads, 1)
    k2_small_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                    SmallArgs a, FwdEpilogue ep, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = aligned_smem(smem_raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);
    uint64_t* empty = full + kMaxStages;
    uint64_t* wready = empty + kMaxStages;  // W4: the int8 tile expanded
    uint64_t* accf = wready + kMaxStages;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(accf + 1);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int S = a.stages;
    const uint32_t rank = cluster_ctarank();
    const int n0 = blockIdx.x * kCh;
    const int kb0 = static_cast<int>((static_cast<long long>(a.kblocks) * rank) / a.S);
    const int kb1 = static_cast<int>((static_cast<long long>(a.kblocks) * (rank + 1)) / a.S);
    const int nkb = kb1 - kb0;
    constexpr uint32_t kWBytes = kCh * 128;
    constexpr uint32_t kPBytes = W4 ? kCh * 64 : 0;
    const uint32_t xbytes = static_cast<uint32_t>(a.MP) * 128;
    const uint32_t stage_bytes = kWBytes + xbytes + kPBytes;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&wready[s], kEpiW);
        }
        mbar_init(accf, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tslot, a.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    pdl_trigger();
    pdl_wait();

    bool ok = true;
    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tmW);
            tma_prefetch_desc(&tmX);
            for (int i = 0; i < nkb; ++i) {
                const int s = i % S;
                if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1, status)) break;
                uint8_t* st = smem + s * stage_bytes;
                mbar_arrive_expect_tx(&full[s], W4 ? xbytes + kPBytes : stage_bytes);
                if constexpr (W4) tma_load_2d(st + kWBytes + xbytes, &tmW, &full[s], (kb0 + i) * 64, n0);
                else tma_load_2d(st, &tmW, &full[s], (kb0 + i) * 128, n0);
                tma_load_2d(st + kWBytes, &tmX, &full[s], (kb0 + i) * 128, 0);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id = idesc_i8(128, a.MP);
            for (int i = 0; i < nkb; ++i) {
                const int s = i % S;
                if (!mbar_wait(&full[s], (i / S) & 1, status) ||
                    (W4 && !mbar_wait(&wready[s], (i / S) & 1, status)))
                    break;
                tc_fence_after();
                const uint32_t wb = smem_u32(smem + s * stage_bytes);
                const uint32_t xb = wb + kWBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = smem_desc(wb + kk * 32, 16, 1024, kLayoutSw128);
                    const uint64_t bd = smem_desc(xb + kk * 32, 16, 1024, kLayoutSw128);
                    mma_i8(tmem, ad, bd, id, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&empty[s]);
            }
            mma_commit(accf);
        }
        __syncwarp();
    } else {
        if constexpr (W4) {
            // expand stage i's packed codes: thread t takes packed chunks t,
            // t + 128, ... (4 per row of 64 bytes = 128 codes)
            const int t = threadIdx.x - 64;
            for (int i = 0; i < nkb && ok; ++i) {
                const int s = i % S;
                if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (i / S) & 1, status))) {
                    ok = false;
                    break;
                }
                uint8_t* wt = smem + s * stage_bytes;
                const uint8_t* pk = wt + kWBytes + xbytes;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = t + u * 128;
                    const int n = e >> 2, p = e & 3;
                    uint4 lo, hi;
                    unpack_int4x32(*reinterpret_cast<const uint4*>(pk + n * 64 + p * 16), lo, hi);
                    uint8_t* row = wt + n * 128;
                    *reinterpret_cast<uint4*>(row + (((2 * p) ^ (n & 7)) << 4)) = lo;
                    *reinterpret_cast<uint4*>(row + (((2 * p + 1) ^ (n & 7)) << 4)) = hi;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&wready[s]);
            }
        }
        {
            // the owner columns' xA rows and row scales, while the MMAs run
            const int Wo = a.MP / a.S;
            float* tab = reinterpret_cast<float*>(smem + kRing);
            const int t = threadIdx.x - 64;
            for (int e = t; e < Wo * (RMAX + 1); e += 32 * kEpiW) {
                const int cl = e / (RMAX + 1), j = e % (RMAX + 1);
                const int m = static_cast<int>(rank) * Wo + cl;
                float v = 0.f;
                if (m < a.M) v = j < RMAX ? (j < ep.r ? __ldg(ep.xA + static_cast<size_t>(m) * ep.r + j) : 0.f)
                                          : __ldg(ep.sx + m);
                tab[e] = v;
            }
        }
        ok = __all_sync(0xffffffffu, ok && mbar_wait(accf, 0, status));
        tc_fence_after();
    }
    // every CTA's accumulator is final and its ring idle
    cluster_sync_all();
    const int W = a.MP / a.S;
    uint32_t* recv = reinterpret_cast<uint32_t*>(smem);
    if (warp >= 2) {
        const int q = warp & 3;  // the TMEM lane quarter this warp may access
        if (nkb > 0 && ok) {
            send_partials(tmem, q, lane, a.MP, W, rank, recv);
        } else {
            // no contraction block (or a failed wait): zeros
            const int row = q * 32 + lane;
            for (int c = 0; c < a.MP; ++c) {
                const int owner = c / W;
                dsmem_st(dsmem_addr(recv + (static_cast<uint32_t>(rank) * W + (c - owner * W)) * kCh + row,
                                    static_cast<uint32_t>(owner)), 0.f);
            }
        }
    }
    cluster_sync_all();
    if (warp >= 2) {
        const int row = (warp & 3) * 32 + lane;
        const int n = n0 + row;
        const bool nok = n < a.N;
        float bj[RMAX];
#pragma unroll
        for (int j = 0; j < RMAX; ++j) bj[j] = (nok && j < ep.r) ? __ldg(ep.B + static_cast<size_t>(j) * a.N + n) : 0.f;
        const float swn = nok ? __ldg(ep.sw + n) : 0.f;
        const float bn = (nok && ep.bias) ? __ldg(ep.bias + n) : 0.f;
        OutT* Y = static_cast<OutT*>(ep.Y);
        const float* tab = reinterpret_cast<const float*>(smem + kRing);
        for (int cl = 0; cl < W; ++cl) {
            const int m = static_cast<int>(rank) * W + cl;
            if (m >= a.M) break;
            int acc = 0;
            for (int qq = 0; qq < a.S; ++qq) acc += static_cast<int>(recv[(qq * W + cl) * kCh + row]);
            if (!nok) continue;
            const float* tr = tab + cl * (RMAX + 1);
            float lora = 0.f;
#pragma unroll
            for (int j = 0; j < RMAX; ++j) lora = fmaf(tr[j], bj[j], lora);
            float y = fmaf(static_cast<float>(acc), __fmul_rn(tr[RMAX], swn), fmaf(ep.c, lora, bn));
            if (ep.relu) y = fmaxf(y, 0.f);
            Y[static_cast<size_t>(m) * a.N + n] = ActIO<OutT>::from_f(y);
            if (ep.acc) ep.acc[static_cast<size_t>(m) * a.N + n] = acc;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, a.tmem_cols);
    }
}

// ------------------------------------------------------------------ dX
// A dX stage: the de-quantized tile (128 output channels k, MN-major, x 64
// contraction rows n; two 64-channel blocks 8 KB apart), then the stage's
// int8 codes as TMA left them ([64 rows n][128 k], no swizzle), then the dY
// tile (MP tokens x 64 n, K-major, 128-byte swizzle).
constexpr uint32_t kDqLbo = 8 * 1024;
constexpr uint32_t kDqTileBytes = kCh * 64 * 2;
constexpr uint32_t kCodeBytes = 64 * kCh;

// W4: packed int4 codes Wp [N, K/2]; a stage's codes are [64 rows][64 bytes].
template <int RMAX, bool W4>
__global__ void __launch_bounds__(kDxThreads, 1)
    k3_small_kernel(const __grid_constant__ CUtensorMap tmDY, const __grid_constant__ CUtensorMap tmW,
                    const float* __restrict__ sw, SmallArgs a, DxEpilogue ep, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = aligned_smem(smem_raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);
    uint64_t* wready = full + kMaxStages;
    uint64_t* empty = wready + kMaxStages;
    uint64_t* accf = empty + kMaxStages;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(accf + 1);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int S = a.stages;
    const uint32_t rank = cluster_ctarank();
    // here the layer's K is the output (channels) and N the contraction
    const int k0 = blockIdx.x * kCh;
    const int nb0 = static_cast<int>((static_cast<long long>(a.kblocks) * rank) / a.S);
    const int nb1 = static_cast<int>((static_cast<long long>(a.kblocks) * (rank + 1)) / a.S);
    const int nnb = nb1 - nb0;
    const uint32_t ybytes = static_cast<uint32_t>(a.MP) * 128;
    constexpr uint32_t kCodes = W4 ? kCodeBytes / 2 : kCodeBytes;
    const uint32_t stage_bytes = kDqTileBytes + kCodeBytes + ybytes;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&wready[s], kDqW);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tslot, a.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    pdl_trigger();
    pdl_wait();

    bool ok = true;
    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tmDY);
            tma_prefetch_desc(&tmW);
            for (int i = 0; i < nnb; ++i) {
                const int s = i % S;
                if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1, status)) break;
                uint8_t* st = smem + s * stage_bytes + kDqTileBytes;
                mbar_arrive_expect_tx(&full[s], kCodes + ybytes);
                tma_load_2d(st, &tmW, &full[s], W4 ? k0 / 2 : k0, (nb0 + i) * 64);
                tma_load_2d(st + kCodeBytes, &tmDY, &full[s], (nb0 + i) * 64, 0);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id = idesc_bf16(128, a.MP, true, false);
            for (int i = 0; i < nnb; ++i) {
                const int s = i % S;
                if (!mbar_wait(&full[s], (i / S) & 1, status) ||
                    !mbar_wait(&wready[s], (i / S) & 1, status))
                    break;
                tc_fence_after();
                const uint32_t wb = smem_u32(smem + s * stage_bytes);
                const uint32_t yb = wb + kDqTileBytes + kCodeBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = smem_desc(wb + kk * 2048, kDqLbo, 1024, kLayoutSw128);
                    const uint64_t bd = smem_desc(yb + kk * 32, 16, 1024, kLayoutSw128);
                    mma_bf16(tmem, ad, bd, id, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&empty[s]);
            }
            mma_commit(accf);
        }
        __syncwarp();
    } else if (warp < 2 + kDqW) {
        // de-quantize: stage i holds contraction rows n = (nb0 + i) * 64 .. + 63
        // and channels k0 .. k0 + 127 (codes outside the matrix are TMA's
        // zero fill); thread t converts chunks t, t + 256, ... (8 chunks of
        // 16 codes per row).  The stage's bf16 area is free once its codes
        // have landed: the producer refills a stage only after its MMAs.
        const int t = threadIdx.x - 64;
        // 16-byte chunks: 16 int8 codes, or 32 packed int4 codes
        constexpr int kCPR = W4 ? 4 : 8;          // chunks per row
        constexpr int kDqT = 32 * kDqW;           // de-quantize threads
        constexpr int kPer = 64 * kCPR / kDqT;    // chunks per thread
        static_assert(64 * kCPR % kDqT == 0, "chunks per thread");
        constexpr int kSpan = W4 ? 32 : 16;       // channels per chunk
        // the row scales of the next kPD stages are loaded ahead of use
        constexpr int kPD = 4;
        float scr[kPD][kPer];
        auto load_scales = [&](int i, float (&dst)[kPer]) {
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int n = (nb0 + i) * 64 + (t + u * kDqT) / kCPR;
                dst[u] = (i < nnb && n < a.N) ? __ldg(sw + n) : 0.f;
            }
        };
#pragma unroll
        for (int v = 0; v < kPD; ++v) load_scales(v, scr[v]);
        for (int i0 = 0; i0 < nnb && ok; i0 += kPD)
#pragma unroll
        for (int v = 0; v < kPD; ++v) {
            const int i = i0 + v;
            if (i >= nnb) break;
            const int s = i % S;
            if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (i / S) & 1, status))) {
                ok = false;
                break;
            }
            uint8_t* wt = smem + s * stage_bytes;
            const uint8_t* codes = wt + kDqTileBytes;
            uint4 raw[kPer];
            float sc[kPer];
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int c = t + u * kDqT;
                const int nr = c / kCPR, kc = c % kCPR;
                raw[u] = *reinterpret_cast<const uint4*>(codes + nr * (16 * kCPR) + kc * 16);
                sc[u] = scr[v][u];
            }
            load_scales(i + kPD, scr[v]);
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int c = t + u * kDqT;
                const int nr = c / kCPR, kc = c % kCPR;
                const int mn = kc * kSpan;
                uint32_t o[8];
                if constexpr (W4) {
                    uint4 lo, hi;
                    unpack_int4x32(raw[u], lo, hi);
                    dequant16(lo, sc[u], o);
                    *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn, nr, kDqLbo)) = make_uint4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn + 8, nr, kDqLbo)) = make_uint4(o[4], o[5], o[6], o[7]);
                    dequant16(hi, sc[u], o);
                    *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn + 16, nr, kDqLbo)) = make_uint4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn + 24, nr, kDqLbo)) = make_uint4(o[4], o[5], o[6], o[7]);
                } else {
                    dequant16(raw[u], sc[u], o);
                    *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn, nr, kDqLbo)) = make_uint4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn + 8, nr, kDqLbo)) = make_uint4(o[4], o[5], o[6], o[7]);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&wready[s]);
        }
        __syncwarp();
    } else {
        {
            // the owner columns' G rows (c G), while the MMAs run
            const int Wo = a.MP / a.S;
            float* tab = reinterpret_cast<float*>(smem + kRing);
            const int t = threadIdx.x - 32 * (2 + kDqW);
            for (int e = t; e < Wo * RMAX; e += 32 * kEpiW) {
                const int cl = e / RMAX, j = e % RMAX;
                const int m = static_cast<int>(rank) * Wo + cl;
                tab[e] = (m < a.M && j < ep.r) ? ep.c * g_row(ep, a.M, m, j) : 0.f;
            }
        }
        ok = __all_sync(0xffffffffu, mbar_wait(accf, 0, status));
        tc_fence_after();
    }
    cluster_sync_all();
    const int W = a.MP / a.S;
    uint32_t* recv = reinterpret_cast<uint32_t*>(smem);
    constexpr int kEpi0 = 2 + kDqW;
    if (warp >= kEpi0) {
        const int q = warp & 3;  // the TMEM lane quarter this warp may access
        if (nnb > 0 && ok) {
            send_partials(tmem, q, lane, a.MP, W, rank, recv);
        } else {
            const int row = q * 32 + lane;
            for (int c = 0; c < a.MP; ++c) {
                const int owner = c / W;
                dsmem_st(dsmem_addr(recv + (static_cast<uint32_t>(rank) * W + (c - owner * W)) * kCh + row,
                                    static_cast<uint32_t>(owner)), 0.f);
            }
        }
    }
    cluster_sync_all();
    if (warp >= kEpi0) {
        const int row = (warp & 3) * 32 + lane;
        const int k = k0 + row;
        const bool kok = k < a.K;
        float aj[RMAX];
#pragma unroll
        for (int j = 0; j < RMAX; ++j) aj[j] = (kok && j < ep.r) ? a_at(ep, k, j) : 0.f;
        __nv_bfloat16* dX = static_cast<__nv_bfloat16*>(ep.dX);
        const __nv_bfloat16* gate = static_cast<const __nv_bfloat16*>(ep.gate);
        const float* tab = reinterpret_cast<const float*>(smem + kRing);
        for (int cl = 0; cl < W; ++cl) {
            const int m = static_cast<int>(rank) * W + cl;
            if (m >= a.M) break;
            float acc = 0.f;
            for (int qq = 0; qq < a.S; ++qq) acc += __uint_as_float(recv[(qq * W + cl) * kCh + row]);
            if (!kok) continue;
            const float* tr = tab + cl * RMAX;
            float l = 0.f;
#pragma unroll
            for (int j = 0; j < RMAX; ++j) l = fmaf(tr[j], aj[j], l);
            float y = acc + l;
            if (gate && !(__bfloat162float(gate[static_cast<size_t>(m) * a.K + k]) > 0.f)) y = 0.f;
            dX[static_cast<size_t>(m) * a.K + k] = __float2bfloat16_rn(y);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, a.tmem_cols);
    }
}

uint32_t pow2_cols(int mp) {
    uint32_t c = 32;
    while (c < static_cast<uint32_t>(mp)) c <<= 1;
    return c;
}

// The split: the largest power of two <= kMaxSplit with at most one wave of
// CTAs and at least two contraction blocks per CTA.
int pick_split(int tiles, int kblocks) {
    int s = 1;
    while (2 * s <= kMaxSplit && tiles * 2 * s <= sm_count() && 2 * (2 * s) <= kblocks) s *= 2;
    return s;
}

}  // namespace

bool small_m_applies(int M, int out_channels, int r) {
    if (M < 1 || M > kMaxTokens || r > 16) return false;
    // only where the large-tile kernels leave SMs idle
    return ((M + 127) / 128) * ((out_channels + 127) / 128) < sm_count();
}

cudaError_t launch_gemm_i8_fwd_small(Act act, const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                                     const FwdEpilogue& ep, int* status, cudaStream_t s, bool w4) {
    SmallArgs a{};
    a.M = M;
    a.N = N;
    a.K = K;
    a.MP = (M + 15) / 16 * 16;
    a.kblocks = (K + 127) / 128;
    const int tiles = (N + kCh - 1) / kCh;
    a.S = pick_split(tiles, a.kblocks);
    const uint32_t stage = kCh * 128 + static_cast<uint32_t>(a.MP) * 128 + (w4 ? kCh * 64 : 0);
    a.stages = static_cast<int>(kRing / stage) > kMaxStages ? kMaxStages : static_cast<int>(kRing / stage);
    a.tmem_cols = pow2_cols(a.MP);
    CUtensorMap tw, tx;
    const bool wok = w4 ? make_tmap_2d(&tw, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, K / 2, kCh, 64,
                                       CU_TENSOR_MAP_SWIZZLE_NONE)
                        : make_tmap_2d(&tw, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, K, kCh, 128,
                                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (!wok ||
        !make_tmap_2d(&tx, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K, K, a.MP, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const size_t smem = kBarOff + 1024 + 256;
    const dim3 grid(tiles, a.S);
    auto run = [&](auto kern) -> cudaError_t {
        cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        return launch_k(kern, grid, dim3(kFwdThreads), smem, s, a.S, tw, tx, a, ep, status);
    };
    auto by_w4 = [&](auto k8, auto k4) { return w4 ? run(k4) : run(k8); };
    if (act == kBF16) {
        if (ep.r <= 4) return by_w4(k2_small_kernel<__nv_bfloat16, 4, false>, k2_small_kernel<__nv_bfloat16, 4, true>);
        if (ep.r <= 8) return by_w4(k2_small_kernel<__nv_bfloat16, 8, false>, k2_small_kernel<__nv_bfloat16, 8, true>);
        return by_w4(k2_small_kernel<__nv_bfloat16, 16, false>, k2_small_kernel<__nv_bfloat16, 16, true>);
    }
    if (ep.r <= 4) return by_w4(k2_small_kernel<float, 4, false>, k2_small_kernel<float, 4, true>);
    if (ep.r <= 8) return by_w4(k2_small_kernel<float, 8, false>, k2_small_kernel<float, 8, true>);
    return by_w4(k2_small_kernel<float, 16, false>, k2_small_kernel<float, 16, true>);
}

cudaError_t launch_gemm_dx_small(const void* dY, const int8_t* Wq, const float* sw, int M, int N, int K,
                                 const DxEpilogue& ep, int* status, cudaStream_t s, bool w4) {
    SmallArgs a{};
    a.M = M;
    a.N = N;
    a.K = K;
    a.MP = (M + 15) / 16 * 16;
    a.kblocks = (N + 63) / 64;
    const int tiles = (K + kCh - 1) / kCh;
    a.S = pick_split(tiles, a.kblocks);
    const uint32_t stage = kDqTileBytes + kCodeBytes + static_cast<uint32_t>(a.MP) * 128;
    a.stages = static_cast<int>(kRing / stage) > kMaxStages ? kMaxStages : static_cast<int>(kRing / stage);
    a.tmem_cols = pow2_cols(a.MP);
    CUtensorMap ty, tw;
    if (!make_tmap_2d(&ty, dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, static_cast<uint64_t>(N) * 2, a.MP,
                      64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !(w4 ? make_tmap_2d(&tw, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, K / 2, 64, kCh / 2,
                            CU_TENSOR_MAP_SWIZZLE_NONE)
             : make_tmap_2d(&tw, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, K, 64, kCh,
                            CU_TENSOR_MAP_SWIZZLE_NONE)))
        return cudaErrorInvalidValue;
    const size_t smem = kBarOff + 1024 + 256;
    const dim3 grid(tiles, a.S);
    auto run = [&](auto kern) -> cudaError_t {
        cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        return launch_k(kern, grid, dim3(kDxThreads), smem, s, a.S, ty, tw, sw, a, ep, status);
    };
    if (ep.r <= 4) return w4 ? run(k3_small_kernel<4, true>) : run(k3_small_kernel<4, false>);
    if (ep.r <= 8) return w4 ? run(k3_small_kernel<8, true>) : run(k3_small_kernel<8, false>);
    return w4 ? run(k3_small_kernel<16, true>) : run(k3_small_kernel<16, false>);
}

}  // namespace qlora
