// k2_gemm_i8.cu -- forward int8 GEMM of the int8-LoRA Dense layer on the
// 5th-generation tensor cores, with the whole layer epilogue fused:
//
//   acc[m,n]  = sum_k Xq[m,k] Wq[n,k]                          (int32, TMEM)
//   lora[m,n] = sum_j (c xA[m,j]) B[j,n] + 1 * bias[n]          (fp32, TMEM)
//   Y[m,n]    = acc * sx[m] * sw[n] + lora[m,n]
//
// ("Introduce QLoRA-like technique", Results: int8 Dense needs a hardware
// int8 matmul; "Parameter-efficient fine-tuning of GPT-2 with LoRA", "LoRA
// equation" for the added low-rank term, with xA = x . A from the input pass.)
// The rank-r term and the bias are one more small product, [c xA | 1] x
// [B ; bias], issued as tf32 MMAs into a second TMEM accumulator (split into
// tf32 head and remainder for fp32 outputs, which keeps fp32 accuracy).
//
// Persistent kernel, one CTA per SM, 10 warps:
//   warp 0      TMA producer: Xq [128 x 128] and Wq [BN x 128] int8 tiles
//               (128B swizzle, K-major) into a STAGES-deep ring
//   warp 1      TMEM owner and MMA issuer: tcgen05.mma.kind::i8, M=128,
//               N=BN, K=32, then the tf32 rank-r MMAs; two accumulator
//               buffers so that tile i+1's main loop overlaps tile i's
//               epilogue
//   warps 2..9  epilogue: write the tile's rank-r operand tables, then two
//               warps per TMEM lane quarter, each one half of the columns:
//               y = acc * (sx sw) + lora, staged coalesced 16-byte stores
// Ragged M, N, K: the tensor maps zero-fill, the stores are predicated.
#include "internal.h"
#include "ptx.cuh"
#include "tile_epilogue.cuh"

namespace qlora {

namespace {

constexpr int kBM = 128;
constexpr int kBlkK = 128;        // int8 elements per 128-byte swizzle row (one TMA block)
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kUnpackWarps = 4;  // packed int4 kernels: warps that expand the codes per stage

template <bool W4>
__host__ __device__ constexpr int k2_threads() { return kThreads + (W4 ? 32 * kUnpackWarps : 0); }
constexpr int kSmemLimit = 232448;  // 227 KB opt-in dynamic shared memory

template <int BN, typename OutT, int RMAX, bool SPLIT = false, bool W4 = false>
struct K2Cfg {
    static constexpr bool kLoraMMA = RMAX <= 16;
    static constexpr bool kSplit = sizeof(OutT) == 4;      // 3 x tf32 for fp32 outputs
    static constexpr int kKL = ((RMAX + 1 + 7) / 8) * 8;   // [c xA | 1] width
    static constexpr int kTerms = kSplit ? 2 : 1;          // head (+ remainder) tables
    static constexpr int kXtBytes = kLoraMMA ? kBM * kKL * 4 : 0;
    static constexpr int kBtBytes = kLoraMMA ? BN * kKL * 4 : 0;
    static constexpr int kBufBytes = kTerms * (kXtBytes + kBtBytes) + BN * 4 * 2;  // + sw, bias
    static constexpr int kStgBytes = kEpiWarps * 32 * stage_pitch<OutT>();
    // split-K: the partial accumulators of this CTA's rows from every CTA of
    // the cluster, [S][128 / S rows][BN] int32, rows padded by 16 bytes
    // (conflict-free 16-byte accesses by per-lane rows)
    static constexpr int kRedPitch = BN + 4;
    static constexpr int kRedBytes = SPLIT ? kBM * kRedPitch * 4 : 0;
    static constexpr int kFixed = kStgBytes + 2 * kBufBytes + kRedBytes + 512 + 1024;
    // k per stage: two 128-byte blocks (one 3-D TMA box per operand) where
    // two such stages fit, else one
    // (packed int4 kernels: the stage also holds the packed codes, BN x kBK/2)
    static constexpr int kBlk =
        (kSmemLimit - kFixed) / ((kBM + BN + (W4 ? BN / 2 : 0)) * 2 * kBlkK) >= 2 ? 2 : 1;
    static constexpr int kBK = kBlk * kBlkK;
    static constexpr int kABytes = kBM * kBK;
    static constexpr int kBBytes = BN * kBK;
    static constexpr int kPBytes = W4 ? BN * kBK / 2 : 0;
    static constexpr int kStageBytes = kABytes + kBBytes + kPBytes;
    static constexpr int kStagesFit = (kSmemLimit - kFixed) / kStageBytes;
    static constexpr int STAGES = kStagesFit > 8 ? 8 : kStagesFit;
    static_assert(STAGES >= 2, "shared memory budget");
    static constexpr int kStgOff = STAGES * kStageBytes;
    static constexpr int kBufOff = kStgOff + kStgBytes;
    static constexpr int kRedOff = kBufOff + 2 * kBufBytes;
    static constexpr int kBarOff = kRedOff + kRedBytes;
    static constexpr int kTotal = kBarOff + 512 + 1024;
    static constexpr uint32_t kAccCols = 2 * BN;             // int32 acc + fp32 rank-r acc
    // split-K CTAs take one tile each: one accumulator buffer
    static constexpr uint32_t kTmemCols = SPLIT ? kAccCols : 2 * kAccCols;
    static_assert(kTmemCols <= 512, "TMEM");
};

// W4: the kernel is packed int4 codes Wp [N, K/2] (two per byte, even k in
// the low nibble) instead of int8 codes; tmB then maps Wp, and the TMA brings
// each stage's packed tile ([BN rows][kBK/2 bytes], no swizzle) with the Xq
// tile.  Warps 10..13 expand it into the int8 tile the TMA would have written
// for int8 codes (128B swizzle, K-major), and the MMA waits for them as well.
//
// SPLIT: split-K for grids that would leave SMs idle.  The grid is tiles x S
// (S = 2, 4 or 8) with clusters of the S CTAs of one tile (along y); CTA s
// runs k-blocks [s nkb / S, (s+1) nkb / S) of its tile.  Rows
// [s 128/S, (s+1) 128/S) of the tile belong to CTA s: every CTA stores its
// int32 partial of those rows into CTA s's shared memory (distributed shared
// memory, one slot per CTA) and arrives on CTA s's barrier; CTA s adds the S
// slots (in slot order) and runs the epilogue of its rows.  Every CTA issues
// the rank-r MMAs of the whole tile (a few tf32 MMAs) and uses its rows.
template <int BN, typename OutT, int RMAX, bool W4, bool SPLIT>
__global__ void __launch_bounds__(k2_threads<W4>(), 1)
    k2_gemm_i8_lora_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB, int k3d, int M, int N, int K,
                           const uint8_t* __restrict__ Wp, FwdEpilogue ep, int* status) {
    using C = K2Cfg<BN, OutT, RMAX, SPLIT, W4>;
    static_assert(!(SPLIT && W4), "split-K runs on int8 codes");
    constexpr int S = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;    // [2]
    uint64_t* tempty = tfull + 2;   // [2]
    uint64_t* lready = tempty + 2;  // [2] rank-r operand tables written
    uint64_t* wready = lready + 2;  // [S] packed int4 kernels: the stage's int8 codes written
    uint64_t* rbar = wready + S;    // split-K leader: every CTA's partial has been added
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rbar + 1);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int num_n = (N + BN - 1) / BN;
    const int tiles = ((M + kBM - 1) / kBM) * num_n;
    const int nkb = (K + C::kBK - 1) / C::kBK;
    const int split = SPLIT ? static_cast<int>(blockIdx.y) : 0;
    const int nsplit = SPLIT ? static_cast<int>(gridDim.y) : 1;
    const int kb0 = split * nkb / nsplit;
    const int kb1 = (split + 1) * nkb / nsplit;
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kEpiWarps);
            mbar_init(&lready[b], 1);
        }
        if constexpr (W4)
            for (int s = 0; s < S; ++s) mbar_init(&wready[s], kUnpackWarps);
        if constexpr (SPLIT) mbar_init(rbar, 2u * kBM);  // every CTA: its rows' partials, two column halves
        fence_mbar_init();
    }

    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // split-K: no CTA stores into another's slots before that CTA's barrier
    // is initialised (every warp waits on this arrival once, below)
    if constexpr (SPLIT) cluster_arrive();
    pdl_wait();  // the prologue above touched no global memory

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            int g = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int m0 = (t / num_n) * kBM;
                const int n0 = (t % num_n) * BN;
                for (int kb = kb0; kb < kb1; ++kb, ++g) {
                    const int s = g % S;
                    if (g >= S && !mbar_wait(&empty[s], ((g / S) - 1) & 1, status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + s * C::kStageBytes;
                    mbar_arrive_expect_tx(&full[s], W4 ? C::kABytes + C::kPBytes : C::kStageBytes);
                    if constexpr (W4)
                        tma_load_2d(sa + C::kABytes + C::kBBytes, &tmB, &full[s], kb * (C::kBK / 2), n0);
                    // each operand's two k-blocks, consecutive in shared memory
                    if (k3d) {
                        tma_load_3d(sa, &tmA, &full[s], 0, m0, kb * C::kBlk);
                        if constexpr (!W4) tma_load_3d(sa + C::kABytes, &tmB, &full[s], 0, n0, kb * C::kBlk);
                    } else {
#pragma unroll
                        for (int b = 0; b < C::kBlk; ++b) {
                            tma_load_2d(sa + b * (kBM * kBlkK), &tmA, &full[s], (kb * C::kBlk + b) * kBlkK,
                                        m0);
                            if constexpr (!W4)
                                tma_load_2d(sa + C::kABytes + b * (BN * kBlkK), &tmB, &full[s],
                                            (kb * C::kBlk + b) * kBlkK, n0);
                        }
                    }
                }
            }
        }
        __syncwarp();
        if constexpr (SPLIT) cluster_wait();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kBM, BN);
            int g = 0, i = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++i) {
                const int ab = i & 1;
                const int use = i >> 1;
                if (use > 0 && !mbar_wait(&tempty[ab], (use - 1) & 1, status)) break;
                tc_fence_after();
                const uint32_t dacc = tmem + ab * C::kAccCols;
                for (int kb = kb0; kb < kb1; ++kb, ++g) {
                    const int s = g % S;
                    if (!mbar_wait(&full[s], (g / S) & 1, status) ||
                        (W4 && !mbar_wait(&wready[s], (g / S) & 1, status))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + s * C::kStageBytes);
                    const uint32_t b_base = a_base + C::kABytes;
#pragma unroll
                    for (int kk = 0; kk < C::kBK / 32; ++kk) {
                        // 32-byte step kk: block kk / 4, 32 bytes per step within it
                        const uint64_t ad = smem_desc(a_base + (kk >> 2) * (kBM * kBlkK) + (kk & 3) * 32, 16,
                                                      1024, kLayoutSw128);
                        const uint64_t bd = smem_desc(b_base + (kk >> 2) * (BN * kBlkK) + (kk & 3) * 32, 16,
                                                      1024, kLayoutSw128);
                        mma_i8(dacc, ad, bd, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
                    }
                    mma_commit(&empty[s]);
                }
                if constexpr (C::kLoraMMA) {
                    // [c xA | 1] x [B ; bias] into the fp32 accumulator
                    if (ok && !mbar_wait(&lready[ab], use & 1, status)) ok = false;
                    if (ok) {
                        tc_fence_after();
                        constexpr uint32_t tdesc = idesc_tf32(kBM, BN);
                        constexpr uint32_t kSbo = (C::kKL / 4) * 128;
                        const uint32_t buf = smem_u32(smem + C::kBufOff + ab * C::kBufBytes);
                        const uint32_t xt_hi = buf;
                        const uint32_t bt_hi = buf + C::kXtBytes;
                        const uint32_t xt_lo = buf + C::kXtBytes + C::kBtBytes;
                        const uint32_t bt_lo = xt_lo + C::kXtBytes;
                        const uint32_t dl = dacc + BN;
#pragma unroll
                        for (int ks = 0; ks < C::kKL / 8; ++ks) {
                            const uint32_t o = ks * 256;
                            mma_tf32(dl, smem_desc(xt_hi + o, 128, kSbo, kLayoutNone),
                                     smem_desc(bt_hi + o, 128, kSbo, kLayoutNone), tdesc, ks != 0);
                            if constexpr (C::kSplit) {
                                mma_tf32(dl, smem_desc(xt_hi + o, 128, kSbo, kLayoutNone),
                                         smem_desc(bt_lo + o, 128, kSbo, kLayoutNone), tdesc, 1);
                                mma_tf32(dl, smem_desc(xt_lo + o, 128, kSbo, kLayoutNone),
                                         smem_desc(bt_hi + o, 128, kSbo, kLayoutNone), tdesc, 1);
                            }
                        }
                    }
                }
                if (ok) mma_commit(&tfull[ab]);
            }
        }
        __syncwarp();
        if constexpr (SPLIT) cluster_wait();
    } else if (W4 && warp >= 2 + kEpiWarps) {
        // ------------------------------------------------------ int4 unpack
        // Stage g's Wq tile, as the TMA would have written it: k-block b of
        // row n at b * BN * 128 + n * 128, its 16-byte chunk c at position
        // c ^ (n % 8).  One packed 16-byte chunk (32 codes) gives int8 chunks
        // 2p and 2p + 1 of a row; outside the matrix the TMA's zero fill gives
        // zero codes.  The stage's int8 area is free once its packed codes
        // have landed: the producer refills a stage only after its MMAs.
        const int ut = (warp - 2 - kEpiWarps) * 32 + lane;
        constexpr int kPerRow = C::kBlk * 4;  // packed chunks of one row per stage
        constexpr int kItems = BN * kPerRow;
        constexpr int kPer = kItems / (32 * kUnpackWarps);
        static_assert(kItems % (32 * kUnpackWarps) == 0, "packed chunks per unpack thread");
        (void)Wp;
        int g = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            for (int kb = kb0; kb < kb1; ++kb, ++g) {
                const int s = g % S;
                if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (g / S) & 1, status))) {
                    ok = false;
                    break;
                }
                uint8_t* wb = smem + s * C::kStageBytes + C::kABytes;
                const uint8_t* pk = wb + C::kBBytes;
                uint4 raw[kPer];
#pragma unroll
                for (int i = 0; i < kPer; ++i) {
                    const int e = ut + i * 32 * kUnpackWarps;
                    const int n = e / kPerRow;
                    const int rem = e % kPerRow;
                    raw[i] = *reinterpret_cast<const uint4*>(pk + n * (C::kBK / 2) + (rem / 4) * 64 + (rem % 4) * 16);
                }
#pragma unroll
                for (int i = 0; i < kPer; ++i) {
                    const int e = ut + i * 32 * kUnpackWarps;
                    const int n = e / kPerRow;
                    const int rem = e % kPerRow;
                    const int p = rem % 4;
                    uint4 lo, hi;
                    unpack_int4x32(raw[i], lo, hi);
                    uint8_t* row = wb + (rem / 4) * (BN * kBlkK) + n * kBlkK;
                    *reinterpret_cast<uint4*>(row + (((2 * p) ^ (n & 7)) << 4)) = lo;
                    *reinterpret_cast<uint4*>(row + (((2 * p + 1) ^ (n & 7)) << 4)) = hi;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&wready[s]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int ew = warp - 2;            // 0 .. 7
        const int q = warp & 3;             // TMEM lane quarter of this warp
        const int half = ew >> 2;           // column half
        const int et = threadIdx.x - 64;    // 0 .. 255
        uint8_t* stg = smem + C::kStgOff + ew * 32 * stage_pitch<OutT>();
        const bool vec = ((static_cast<size_t>(N) * sizeof(OutT)) % 16) == 0;
        OutT* Y = static_cast<OutT*>(ep.Y);
        int i = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
            const int ab = i & 1;
            const int use = i >> 1;
            const int m0 = (t / num_n) * kBM;
            const int n0 = (t % num_n) * BN;
            uint8_t* buf = smem + C::kBufOff + ab * C::kBufBytes;
            float* s_sw = reinterpret_cast<float*>(buf + C::kTerms * (C::kXtBytes + C::kBtBytes));
            float* s_bias = s_sw + BN;
            // ---- this tile's tables (buffer ab was last read two tiles ago) ----
            for (int c = et; c < BN; c += 32 * kEpiWarps) {
                const int n = n0 + c;
                s_sw[c] = n < N ? ep.sw[n] : 0.f;
                s_bias[c] = (n < N && ep.bias) ? ep.bias[n] : 0.f;
            }
            if constexpr (C::kLoraMMA) {
                uint8_t* xt = buf;
                uint8_t* bt = buf + C::kXtBytes;
                uint8_t* xt_lo = buf + C::kXtBytes + C::kBtBytes;
                uint8_t* bt_lo = xt_lo + C::kXtBytes;
                for (int e = et; e < kBM * C::kKL; e += 32 * kEpiWarps) {
                    const int rr = e / C::kKL, j = e % C::kKL;
                    const int m = m0 + rr;
                    float x = 0.f;
                    if (m < M) x = j < ep.r ? ep.xA[static_cast<size_t>(m) * ep.r + j] * ep.c
                                            : (j == ep.r ? 1.f : 0.f);
                    float hi, lo;
                    tf32_split(x, hi, lo);
                    const uint32_t off = kmajor_tf32_offset(rr, j, C::kKL);
                    *reinterpret_cast<float*>(xt + off) = hi;
                    if constexpr (C::kSplit) *reinterpret_cast<float*>(xt_lo + off) = lo;
                }
                for (int e = et; e < BN * C::kKL; e += 32 * kEpiWarps) {
                    const int cc = e / C::kKL, j = e % C::kKL;
                    const int n = n0 + cc;
                    float b = 0.f;
                    if (n < N) b = j < ep.r ? ep.B[static_cast<size_t>(j) * N + n]
                                            : ((j == ep.r && ep.bias) ? ep.bias[n] : 0.f);
                    float hi, lo;
                    tf32_split(b, hi, lo);
                    const uint32_t off = kmajor_tf32_offset(cc, j, C::kKL);
                    *reinterpret_cast<float*>(bt + off) = hi;
                    if constexpr (C::kSplit) *reinterpret_cast<float*>(bt_lo + off) = lo;
                }
                fence_proxy_async_smem();
            }
            named_bar_sync(1, 32 * kEpiWarps);
            if constexpr (C::kLoraMMA) {
                if (et == 0) mbar_arrive(&lready[ab]);
            }

            const int row0 = m0 + q * 32;
            const int row = row0 + lane;
            const bool row_ok = row < M;
            const float sxm = row_ok ? ep.sx[row] : 0.f;
            float xa[C::kLoraMMA ? 1 : RMAX];
            if constexpr (!C::kLoraMMA) {
#pragma unroll
                for (int j = 0; j < RMAX; ++j)
                    xa[j] = (row_ok && j < ep.r) ? ep.xA[static_cast<size_t>(row) * ep.r + j] * ep.c : 0.f;
            }

            bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[ab], use & 1, status));
            tc_fence_after();
            const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + ab * C::kAccCols;
            // split-K: this CTA's rows of the tile and where this lane's row lives
            const int R = kBM / nsplit;
            const int trow = q * 32 + lane;
            const int own_lo = split * R;
            int* slots = reinterpret_cast<int*>(smem + C::kRedOff);
            if constexpr (SPLIT) {
                cluster_wait();
                const int owner = trow / R;
                const uint32_t dst = dsmem_addr(slots + (split * R + trow % R) * C::kRedPitch,
                                                static_cast<uint32_t>(owner));
                if (ok) {
#pragma unroll 1
                    for (int col = half * (BN / 2); col < (half + 1) * (BN / 2); col += kEpiCols) {
                        uint32_t v[kEpiCols];
                        tmem_ld16(tbase + col, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < kEpiCols; e += 4)
                            dsmem_st_v4(dst + 4u * static_cast<uint32_t>(col + e), v[e], v[e + 1], v[e + 2],
                                        v[e + 3]);
                    }
                }
                tc_fence_before();
                mbar_arrive_remote(dsmem_addr(rbar, static_cast<uint32_t>(owner)));
                // every CTA's slots of this CTA's rows have landed
                ok = __all_sync(0xffffffffu, mbar_wait_cluster(rbar, 0, status) && ok);
                tc_fence_after();
                if (own_lo >= q * 32 + 32 || own_lo + R <= q * 32) break;  // no rows of mine here
            }
            if (!ok) break;
            const int row_min = SPLIT ? m0 + own_lo : 0;
            const int row_lim = SPLIT ? min(M, m0 + own_lo + R) : M;
            const bool own_row = !SPLIT || (trow >= own_lo && trow < own_lo + R);
#pragma unroll 1
            for (int col = half * (BN / 2); col < (half + 1) * (BN / 2); col += kEpiCols) {
                uint32_t v[kEpiCols];
                uint32_t l[kEpiCols];
                if constexpr (SPLIT) {
                    // the S partials of this row, added in slot order
#pragma unroll
                    for (int e = 0; e < kEpiCols; ++e) v[e] = 0u;
                    if (own_row) {
                        for (int sp = 0; sp < nsplit; ++sp) {
                            const uint4* p = reinterpret_cast<const uint4*>(
                                slots + (sp * R + trow - own_lo) * C::kRedPitch + col);
#pragma unroll
                            for (int e4 = 0; e4 < kEpiCols / 4; ++e4) {
                                const uint4 w = p[e4];
                                v[4 * e4 + 0] += w.x;
                                v[4 * e4 + 1] += w.y;
                                v[4 * e4 + 2] += w.z;
                                v[4 * e4 + 3] += w.w;
                            }
                        }
                    }
                } else {
                    tmem_ld16(tbase + col, v);
                }
                if constexpr (C::kLoraMMA) tmem_ld16(tbase + BN + col, l);
                tmem_ld_wait();
                float y[kEpiCols];
                const float4* sw4 = reinterpret_cast<const float4*>(s_sw + col);
#pragma unroll
                for (int e4 = 0; e4 < kEpiCols / 4; ++e4) {
                    const float4 w4 = sw4[e4];
                    const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int e = 4 * e4 + u;
                        const float a = static_cast<float>(static_cast<int32_t>(v[e]));
                        if constexpr (C::kLoraMMA) {
                            y[e] = fmaf(a * sxm, wv[u], __uint_as_float(l[e]));
                        } else {
                            const int c = col + e;
                            const int n = n0 + c;
                            float acc = fmaf(a * sxm, wv[u], s_bias[c]);
                            if (n < N)
                                for (int j = 0; j < ep.r; ++j)
                                    acc = fmaf(xa[j], __ldg(ep.B + static_cast<size_t>(j) * N + n), acc);
                            y[e] = acc;
                        }
                    }
                }
                if (ep.relu) {
#pragma unroll
                    for (int e = 0; e < kEpiCols; ++e) y[e] = y[e] > 0.f ? y[e] : 0.f;
                }
                if (ep.acc && row_ok && own_row) {
                    for (int e = 0; e < kEpiCols; ++e)
                        if (n0 + col + e < N)
                            ep.acc[static_cast<size_t>(row) * N + n0 + col + e] = static_cast<int32_t>(v[e]);
                }
                store_block<OutT>(stg, y, lane, Y, static_cast<size_t>(N), row0, row_lim, n0 + col, N, vec,
                                  row_min);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[ab]);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int BN, typename OutT, int RMAX, bool W4, bool SPLIT = false>
cudaError_t launch_cfg(const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                       const FwdEpilogue& ep, int* status, cudaStream_t s, int nsplit = 1) {
    using C = K2Cfg<BN, OutT, RMAX, SPLIT, W4>;
    // Xq and Wq as [row][k-block of 128][128] (one 3-D box per operand and
    // stage) when K splits into whole blocks, else one 2-D box per block
    CUtensorMap ta, tb;
    const int k3d = (K % kBlkK) == 0 ? 1 : 0;
    bool ok;
    // (packed int4 kernels: tmB maps the packed codes [N, K/2], one box of
    // [BN rows][kBK/2 bytes] per stage)
    if (k3d)
        ok = make_tmap_3d_blocks(&ta, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K, kBlkK, kBM, C::kBlk) &&
             (W4 || make_tmap_3d_blocks(&tb, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, kBlkK, BN, C::kBlk));
    else
        ok = make_tmap_2d(&ta, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K, K, kBM, kBlkK,
                          CU_TENSOR_MAP_SWIZZLE_128B) &&
             (W4 || make_tmap_2d(&tb, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, K, BN, kBlkK,
                                 CU_TENSOR_MAP_SWIZZLE_128B));
    if (W4)
        ok = ok && make_tmap_2d(&tb, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, K / 2, BN, C::kBK / 2,
                                CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return cudaErrorInvalidValue;
    auto kern = k2_gemm_i8_lora_kernel<BN, OutT, RMAX, W4, SPLIT>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), C::kTotal);
    if (e != cudaSuccess) return e;
    const int tiles = ((M + kBM - 1) / kBM) * ((N + BN - 1) / BN);
    if constexpr (SPLIT)
        return launch_k(kern, dim3(tiles, nsplit), dim3(k2_threads<W4>()), C::kTotal, s, nsplit, ta, tb,
                        k3d, M, N, K, static_cast<const uint8_t*>(nullptr), ep, status);
    const int grid = tiles < sm_count() ? tiles : sm_count();
    return launch_k(kern, dim3(grid), dim3(k2_threads<W4>()), C::kTotal, s, 1, ta, tb, k3d, M, N, K,
                    W4 ? reinterpret_cast<const uint8_t*>(Wq) : nullptr, ep, status);
}

template <typename OutT, int RMAX, bool W4>
cudaError_t launch_bn(int bn, const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                      const FwdEpilogue& ep, int* status, cudaStream_t s) {
    if (bn == 128) return launch_cfg<128, OutT, RMAX, W4>(Xq, Wq, M, N, K, ep, status, s);
    return launch_cfg<64, OutT, RMAX, W4>(Xq, Wq, M, N, K, ep, status, s);
}

template <typename OutT, bool W4>
cudaError_t launch_r(int bn, const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                     const FwdEpilogue& ep, int* status, cudaStream_t s) {
    if (ep.r <= 4) return launch_bn<OutT, 4, W4>(bn, Xq, Wq, M, N, K, ep, status, s);
    if (ep.r <= 8) return launch_bn<OutT, 8, W4>(bn, Xq, Wq, M, N, K, ep, status, s);
    if (ep.r <= 16) return launch_bn<OutT, 16, W4>(bn, Xq, Wq, M, N, K, ep, status, s);
    return launch_bn<OutT, 64, W4>(bn, Xq, Wq, M, N, K, ep, status, s);
}

}  // namespace

// Split-K factor for a bf16 layer with very few 128 x 128 tiles: the largest
// power of two (2, 4 or 8: one cluster, and whole slices of the 128 tile
// rows) with tiles x S <= SMs and at least two k-blocks per CTA; 1 = no split.
int fwd_split(int M, int N, int K) {
    using C = K2Cfg<128, __nv_bfloat16, 4, true>;
    const int tiles = ((M + kBM - 1) / kBM) * ((N + 127) / 128);
    const int nkb = (K + C::kBK - 1) / C::kBK;
    // only for grids of at most a ninth of the SMs: in a 33-layer stack of
    // 1024-wide layers (64 tiles) the split measured slower per step
    if (9 * tiles > sm_count()) return 1;
    int sp = 1;
    while (sp < 8 && 2 * sp * tiles <= sm_count() && 2 * (2 * sp) <= nkb) sp *= 2;
    return sp;
}

cudaError_t launch_gemm_i8_fwd(Act act, const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                               const FwdEpilogue& ep, int* status, cudaStream_t s, bool w4) {
    if (small_m_applies(M, N, ep.r)) return launch_gemm_i8_fwd_small(act, Xq, Wq, M, N, K, ep, status, s, w4);
    if (gemm_fwd_pair_applies(act, M, N, K, ep.r))
        return launch_gemm_i8_fwd_pair(Xq, Wq, M, N, K, ep, status, s, w4);
    if (act == kBF16 && !w4 && ep.r <= 16) {
        const int sp = fwd_split(M, N, K);
        if (sp > 1) {
            if (ep.r <= 4)
                return launch_cfg<128, __nv_bfloat16, 4, false, true>(Xq, Wq, M, N, K, ep, status, s, sp);
            if (ep.r <= 8)
                return launch_cfg<128, __nv_bfloat16, 8, false, true>(Xq, Wq, M, N, K, ep, status, s, sp);
            return launch_cfg<128, __nv_bfloat16, 16, false, true>(Xq, Wq, M, N, K, ep, status, s, sp);
        }
    }
    // Tile width: 128 columns unless that leaves SMs without a tile.
    const int mt = (M + kBM - 1) / kBM;
    int bn = mt * ((N + 127) / 128) >= sm_count() ? 128 : 64;
    if (act == kBF16)
        return w4 ? launch_r<__nv_bfloat16, true>(bn, Xq, Wq, M, N, K, ep, status, s)
                  : launch_r<__nv_bfloat16, false>(bn, Xq, Wq, M, N, K, ep, status, s);
    return w4 ? launch_r<float, true>(bn, Xq, Wq, M, N, K, ep, status, s)
              : launch_r<float, false>(bn, Xq, Wq, M, N, K, ep, status, s);
}

}  // namespace qlora
