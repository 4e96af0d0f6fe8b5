// k3_dx.cu -- input gradient of the int8-LoRA Dense layer:
//
//   dX[m,k] = sum_n dY[m,n] * bf16(Wq[n,k] * sw[n]) + c * sum_j G[m,j] A[k,j]
//
// The frozen int8 kernel is de-quantized tile by tile in shared memory right
// before the tensor-core product ("How to fine-tune the 4-bit model?"
// thread: decompress the quantized weights in place, then feed the matrix
// unit; the de-quantization cost is paid per batch, not per input).  The
// input quantizer is passed straight through, so only the de-quantized
// kernel and the LoRA factors enter dX.
//
// tcgen05 path (bf16 activations, N a multiple of 8): persistent, one CTA
// per SM, a tile is (128 * MSUB) rows x BN columns of dX; a stage covers 128
// (MSUB = 1) or 64 (MSUB = 2) rows of the contraction.  Warps:
//   warp 0        TMA producer: one box per stage with all the tile's dY rows
//                 (128B swizzle, K-major; a 3-D view of dY gives two 64-column
//                 blocks in one box when N is a multiple of 64)
//   warps 1..C    MMA issuers (C = 4, or 2): tcgen05.mma.kind::f16 (bf16 in,
//                 fp32 accumulate), M=128, N=BN, K=16.  A tcgen05.mma holds
//                 its issuing thread ~0.1 us whatever its N, so the 128 x 64
//                 and 128 x 128 tiles split every stage's k-steps over C
//                 issuers, each with its own TMEM accumulator, and the 256-row
//                 tiles give each 128-row sub-tile its own issuer; two tile
//                 buffers so tile i+1's main loop overlaps tile i's epilogue.
//                 Warp 1 owns the TMEM allocation.
//   8 warps       de-quantize: load their code chunks (int8, or packed int4
//                 unpacked to int8 first) and row scales
//                 from global memory into registers S stages ahead, and
//                 convert every stage into a bf16 tile laid out as the
//                 MN-major 128B-swizzled B operand
//   4 or 8 warps  epilogue: c G A^T (tf32 MMAs from tables they write), the
//                 accumulators added in chain order, an optional ReLU-backward
//                 gate, staged coalesced stores of dX
// SIMT path: fp32 activations, or rows of dY that the Tensor Memory
// Accelerator cannot describe (N*2 bytes not a multiple of 16).
#include "internal.h"
#include "ptx.cuh"
#include "tile_epilogue.cuh"
#include "dx_common.cuh"

namespace qlora {

namespace {

constexpr int kBlkN = 64;  // one 128-byte swizzle row of bf16: the dY block a 2-D box covers
constexpr int kDqWarps = 8;
constexpr int kSmemLimit = 232448;

template <int MSUB, int BN, int RMAX>
struct K3Cfg {
    static constexpr int kBM = 128 * MSUB;
    // epilogue warps: two per TMEM lane quarter (row sub-tiles, or column
    // halves), one for the 128 x 64 tiles, whose four extra MMA issuers would
    // otherwise leave too few registers per thread
    static constexpr int kEpiWarps = (MSUB == 1 && BN == 64) ? 4 : 8;
    static constexpr int kEpiPerQuarter = kEpiWarps / 4;
    static_assert(MSUB == 1 || kEpiWarps == 8, "one epilogue warp pair per row sub-tile");
    // contraction (n) per stage: 128 (two 64-column dY blocks in one 3-D TMA
    // box), 64 for the 256-row tiles so that two stages fit
    static constexpr int kBKn = MSUB == 2 ? 64 : 128;
    static constexpr int kBlk = kBKn / kBlkN;
    static_assert(MSUB == 1 || kBlk == 1, "one dY box per stage covers the sub-tiles of one block");
    // rank <= 16: c G A^T runs on the tensor cores as tf32 MMAs into the same
    // fp32 accumulator (operand tables c*G [kBM x kKL] and A [BN x kKL] per
    // accumulator buffer); larger ranks fall back to CUDA-core FMAs.
    static constexpr bool kLoraMMA = RMAX <= 16;
    static constexpr int kKL = RMAX <= 8 ? 8 : 16;
    static constexpr int kGtBytes = kLoraMMA ? kBM * kKL * 4 : 0;
    static constexpr int kAtBytes = kLoraMMA ? BN * kKL * 4 : 0;
    static constexpr int kASub = 128 * kBKn * 2;       // one dY sub-tile, bf16
    static constexpr int kABytes = MSUB * kASub;
    static constexpr int kWBytes = kBKn * BN * 2;      // de-quantized bf16 tile
    static constexpr int kStageBytes = kABytes + kWBytes;
    static constexpr int kStgBytes = kEpiWarps * 32 * stage_pitch<__nv_bfloat16>();
    // one set of rank-r operand tables: the epilogue warps write a tile's
    // tables only after the previous tile's accumulator (and with it that
    // tile's rank-r MMAs) is complete, so two sets are never live at once
    static constexpr int kParamBytes = kGtBytes + kAtBytes;
    static constexpr int kFixed = kStgBytes + kParamBytes + 512 + 1024;
    static constexpr int kStagesFit = (kSmemLimit - kFixed) / kStageBytes;
    static constexpr int STAGES = kStagesFit > 8 ? 8 : kStagesFit;
    static_assert(STAGES >= 2, "shared memory budget");
    // de-quantize stage groups: four where the stages divide into them
    static constexpr int kDqGroups = STAGES % 4 == 0 ? 4 : (STAGES % 2 == 0 ? 2 : 1);
    static constexpr int kStgOff = STAGES * kStageBytes;
    static constexpr int kTabOff = kStgOff + kStgBytes;
    static constexpr int kBarOff = kTabOff + kParamBytes;
    static constexpr int kTotal = kBarOff + 512 + 1024;
    // A tcgen05.mma holds its issuing thread ~0.1 us whatever its N, so the
    // contraction of a tile is split over kChains MMA-issuing warps, each with
    // its own TMEM accumulator (added in chain order by the epilogue); two
    // tile buffers of kChains accumulators fill the 512 TMEM columns.
    // The 256-row tiles give each 128-row sub-tile its own issuer instead
    // (kSplitRows): the two sub-tile accumulators are separate already.
    static constexpr int kChains = (MSUB == 1 && BN == 64) ? 4 : 2;
    static constexpr bool kSplitRows = MSUB == 2;
    static constexpr int kKChains = kSplitRows ? 1 : kChains;  // accumulators added by the epilogue
    static constexpr uint32_t kAccCols = MSUB * BN;             // one chain's accumulator
    static constexpr uint32_t kBufCols = kKChains * kAccCols;   // one tile buffer
    static constexpr uint32_t kTmemCols = 2 * kBufCols;
    static_assert(kTmemCols <= 512, "TMEM");
    static_assert(kSplitRows ? kChains == MSUB : (kBKn / 16) % kChains == 0, "work per issuer");
    // warps: producer, kChains MMA issuers, de-quantize, epilogue
    static constexpr int kDqWarp0 = 1 + kChains;
    static constexpr int kEpiWarp0 = kDqWarp0 + kDqWarps;
    static constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
};

// MODE 0: int8 codes [N, K] with a scale per contraction row.  MODE 1: packed
// int4 codes [N, K/2] (two per byte, even k in the low nibble); a 16-byte
// fetch then carries 32 codes.  MODE 2: uint8 affine codes of an
// outlier-compensated kernel (ep.ol), whose fp16 outliers are written over
// the de-quantized tile.
template <int MSUB, int BN, int RMAX, int MODE>
__global__ void __launch_bounds__(K3Cfg<MSUB, BN, RMAX>::kThreads, 1)
    k3_dx_dequant_kernel(const __grid_constant__ CUtensorMap tmDY, int dy3d,
                         const int8_t* __restrict__ Wq, const float* __restrict__ sw, int M, int N,
                         int K, DxEpilogue ep, int* status) {
    using C = K3Cfg<MSUB, BN, RMAX>;
    constexpr int S = C::STAGES;
    constexpr int kBKn = C::kBKn;
    constexpr bool W4 = MODE == 1;
    constexpr uint32_t kLbo = (kBKn / 8) * 1024;  // MN-block stride of the bf16 tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* wready = full + S;
    uint64_t* empty = wready + S;
    uint64_t* tfull = empty + S;   // [2]
    uint64_t* tempty = tfull + 2;  // [2]
    uint64_t* lready = tempty + 2; // [2] rank-r operand tables written
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lready + 2);
    uint8_t* tabs = smem + C::kTabOff;  // c*G table, A table

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int num_k = (K + BN - 1) / BN;
    const int tiles = ((M + C::kBM - 1) / C::kBM) * num_k;
    const int nkb = (N + kBKn - 1) / kBKn;
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&wready[s], kDqWarps / C::kDqGroups);  // the stage group's warps
            mbar_init(&empty[s], C::kChains);  // every MMA issuer, once per use
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], C::kChains);
            mbar_init(&tempty[b], C::kEpiWarps);
            mbar_init(&lready[b], C::kEpiWarps);
        }
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
    pdl_wait();  // the prologue above touched no global memory

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmDY);
            int g = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int m0 = (t / num_k) * C::kBM;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % S;
                    if (g >= S && !mbar_wait(&empty[s], ((g / S) - 1) & 1, status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + s * C::kStageBytes;
                    mbar_arrive_expect_tx(&full[s], C::kABytes);
                    // all kBM rows in one box: the stage's kBlk 64-column blocks
                    // (MSUB == 1), or both 128-row sub-tiles of one block (MSUB
                    // == 2), consecutive in shared memory
                    if (dy3d) {
                        tma_load_3d(sa, &tmDY, &full[s], 0, m0, kb * C::kBlk);
                    } else {
#pragma unroll
                        for (int b = 0; b < C::kBlk; ++b)
                            tma_load_2d(sa + b * (C::kBM * kBlkN * 2), &tmDY, &full[s],
                                        (kb * C::kBlk + b) * kBlkN, m0);
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp < C::kDqWarp0) {
        // ------------------------------------------------------ MMA issuers
        // issuer ch takes the k-steps ch, ch + kChains, ... of every stage
        // into its own accumulator, or (256-row tiles) every k-step of
        // sub-tile ch; each issuer adds the rank-r term of its rows
        const int ch = warp - 1;
        constexpr int kKStep = C::kSplitRows ? 1 : C::kChains;
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, BN, false, true);
            int g = 0, i = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++i) {
                const int ab = i & 1;
                const int use = i >> 1;
                if (use > 0 && !mbar_wait(&tempty[ab], (use - 1) & 1, status)) break;
                tc_fence_after();
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % S;
                    if (!mbar_wait(&full[s], (g / S) & 1, status) ||
                        !mbar_wait(&wready[s], (g / S) & 1, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + s * C::kStageBytes);
                    const uint32_t w_base = a_base + C::kABytes;
#pragma unroll
                    for (int kk = C::kSplitRows ? 0 : ch; kk < kBKn / 16; kk += kKStep) {
                        const uint64_t bd = smem_desc(w_base + kk * 2048, kLbo, 1024, kLayoutSw128);
#pragma unroll
                        for (int ms = 0; ms < MSUB; ++ms) {
                            if (C::kSplitRows && ms != ch) continue;
                            // 16-column step kk: block kk / 4 of the sub-tile, 32 bytes per step within it
                            const uint64_t ad = smem_desc(
                                a_base + ms * C::kASub + (kk >> 2) * (128 * kBlkN * 2) + (kk & 3) * 32, 16,
                                1024, kLayoutSw128);
                            const uint32_t d = C::kSplitRows ? tmem + ab * C::kBufCols + ms * BN
                                                             : tmem + ab * C::kBufCols + ch * C::kAccCols;
                            const bool first = C::kSplitRows ? (kb == 0 && kk == 0) : (kb == 0 && kk == ch);
                            mma_bf16(d, ad, bd, idesc, first ? 0u : 1u);
                        }
                    }
                    mma_commit(&empty[s]);
                }
                if (C::kLoraMMA && (C::kSplitRows || ch == 0)) {
                    // + (c G) A^T: tf32 MMAs from the tables the epilogue warps wrote
                    if (ok && !mbar_wait(&lready[ab], use & 1, status)) ok = false;
                    if (ok) {
                        tc_fence_after();
                        constexpr uint32_t tdesc = idesc_tf32(128, BN);
                        constexpr uint32_t kSbo = (C::kKL / 4) * 128;
                        const uint32_t gt = smem_u32(tabs);
                        const uint32_t at = gt + C::kGtBytes;
#pragma unroll
                        for (int ks = 0; ks < C::kKL / 8; ++ks) {
                            const uint64_t bd = smem_desc(at + ks * 256, 128, kSbo, kLayoutNone);
#pragma unroll
                            for (int ms = 0; ms < MSUB; ++ms) {
                                if (C::kSplitRows && ms != ch) continue;
                                const uint64_t ad =
                                    smem_desc(gt + ms * 16 * kSbo + ks * 256, 128, kSbo, kLayoutNone);
                                mma_tf32(tmem + ab * C::kBufCols + ms * BN, ad, bd, tdesc, 1);
                            }
                        }
                    }
                }
                if (ok) mma_commit(&tfull[ab]);
            }
        }
        __syncwarp();
    } else if (warp < C::kEpiWarp0) {
        // ------------------------------------------------------ de-quantize
        // The eight warps form kDqGroups groups; group q converts the stages
        // g = q, q + kDqGroups, ... (all of a stage's codes), so a warp has
        // kDqGroups stage-times for each of its stages and the pace is set by
        // the warps' throughput, not by the latency of one stage's
        // load-convert-store-signal chain.  The codes and row scales of a
        // group's next S / kDqGroups stages are held in registers (loaded
        // that many group stages ahead); a chunk outside the matrices is
        // zeroed through its scale.  The stage and tile cursors advance
        // without divisions.
        constexpr int kDqGroups = C::kDqGroups;
        constexpr int kWPG = kDqWarps / kDqGroups;
        const int dw = warp - C::kDqWarp0;  // 0 .. 7
        const int grp = dw / kWPG;
        const int gw = dw % kWPG;
        constexpr int kCodes = W4 ? 32 : 16;  // codes per 16-byte chunk
        constexpr int kChunksPerRow = BN / kCodes;
        const size_t row_bytes = W4 ? static_cast<size_t>(K) / 2 : static_cast<size_t>(K);
        constexpr int kChunks = kBKn * kChunksPerRow;
        constexpr int kPerLane = kChunks / (32 * kWPG);
        static_assert(kChunks % (32 * kWPG) == 0, "chunks per stage");
        constexpr int P = S / kDqGroups;  // register ring of a group
        static_assert(S % kDqGroups == 0, "stages per group");
        const int my_tiles = blockIdx.x < tiles ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
        const int total_kb = my_tiles * nkb;
        // fetch cursor: stage g = grp + kDqGroups * j -> (tile ft of this CTA, block fkb)
        int fj = 0, ft = 0, fkb = grp;
        while (fkb >= nkb) { fkb -= nkb; ++ft; }
        int fk0 = ((static_cast<int>(blockIdx.x) + ft * static_cast<int>(gridDim.x)) % num_k) * BN;
        uint4 qr[P][kPerLane];
        float sr[P][kPerLane];
        uint32_t inb[P];  // bit i: chunk i of the ring slot lies inside the matrices
        float ascale = 0.f, abias = 0.f;  // MODE 2: the tensor's affine parameters
        if constexpr (MODE == 2) {
            ascale = __ldg(ep.ol.par + 2);
            abias = __ldg(ep.ol.par + 3);
        }
        auto fetch = [&](uint4 (&q)[kPerLane], float (&sc)[kPerLane], uint32_t& in_bits) {
            const bool live_g = grp + kDqGroups * fj < total_kb;
            in_bits = 0;
#pragma unroll
            for (int i = 0; i < kPerLane; ++i) {
                const int c = gw * 32 + lane + i * 32 * kWPG;
                int cr, cc;
                chunk_rc<kChunksPerRow>(c, cr, cc);
                const int n = fkb * kBKn + cr;
                const int k = fk0 + cc * kCodes;
                if (live_g && n < N && k < K) in_bits |= 1u << i;
                const int nc = n < N ? n : N - 1;
                const int kc = k < K ? k : K - kCodes;
                q[i] = __ldg(reinterpret_cast<const uint4*>(Wq + static_cast<size_t>(nc) * row_bytes +
                                                            (W4 ? kc / 2 : kc)));
                sc[i] = MODE == 2 ? 1.f : __ldg(sw + nc);
            }
            ++fj;
            fkb += kDqGroups;
            bool moved = false;
            while (fkb >= nkb) {
                fkb -= nkb;
                ++ft;
                moved = true;
            }
            if (moved) fk0 = ((static_cast<int>(blockIdx.x) + ft * static_cast<int>(gridDim.x)) % num_k) * BN;
        };
#pragma unroll
        for (int v = 0; v < P; ++v) fetch(qr[v], sr[v], inb[v]);
        bool live = true;
        for (int j0 = 0; live; j0 += P) {
#pragma unroll
            for (int v = 0; v < P; ++v) {
                const int g = grp + kDqGroups * (j0 + v);
                if (g >= total_kb) {
                    live = false;
                    break;
                }
                const int u = grp + kDqGroups * v;  // shared-memory stage: g % S
                if (g >= S &&
                    !__all_sync(0xffffffffu, mbar_wait(&empty[u], ((g / S) - 1) & 1, status))) {
                    live = false;
                    break;
                }
                uint8_t* wt = smem + u * C::kStageBytes + C::kABytes;
#pragma unroll
                for (int i = 0; i < kPerLane; ++i) {
                    const int c = gw * 32 + lane + i * 32 * kWPG;
                    int nr, kc;                          // contraction row, chunk of kCodes columns
                    chunk_rc<kChunksPerRow>(c, nr, kc);
                    const float scale = (inb[v] >> i) & 1u ? sr[v][i] : 0.f;
                    const int mn = kc * kCodes;
                    uint32_t o[8];
                    if constexpr (W4) {
                        uint4 lo, hi;
                        unpack_int4x32(qr[v][i], lo, hi);
                        dequant16(lo, scale, o);
                        *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn, nr, kLbo)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn + 8, nr, kLbo)) =
                            make_uint4(o[4], o[5], o[6], o[7]);
                        dequant16(hi, scale, o);
                        *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn + 16, nr, kLbo)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn + 24, nr, kLbo)) =
                            make_uint4(o[4], o[5], o[6], o[7]);
                    } else {
                        if constexpr (MODE == 2) {
                            // outside the matrices: zero through the affine parameters
                            const bool in = (inb[v] >> i) & 1u;
                            dequant16_affine(qr[v][i], in ? ascale : 0.f, in ? abias : 0.f, o);
                        } else {
                            dequant16(qr[v][i], scale, o);
                        }
                        *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn, nr, kLbo)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn + 8, nr, kLbo)) =
                            make_uint4(o[4], o[5], o[6], o[7]);
                    }
                }
                if constexpr (MODE == 2) {
                    // The warp wrote whole tile rows nr = kRW gw + (c % 32) /
                    // kChunksPerRow + kRW kWPG i (kRW rows per 32 chunks);
                    // its lanes now write those rows' outliers.
                    constexpr int kRW = 32 / kChunksPerRow;
                    __syncwarp();
                    const int t = static_cast<int>(blockIdx.x) + (g / nkb) * static_cast<int>(gridDim.x);
                    const int c0 = (t % num_k) * BN;
                    for (int idx = lane; idx < kPerLane * kRW; idx += 32) {
                        const int nr = gw * kRW + idx % kRW + kRW * kWPG * (idx / kRW);
                        const int n = (g % nkb) * kBKn + nr;
                        if (n < N && c0 < K) patch_outliers(ep.ol, n, c0, BN, wt, nr, kLbo);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&wready[u]);
                fetch(qr[v], sr[v], inb[v]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int ew = warp - C::kEpiWarp0;  // 0 .. 7
        const int q = warp & 3;              // TMEM lane quarter of this warp
        const int sub = ew >> 2;             // MSUB == 2: row sub-tile, else column part
        const int et = threadIdx.x - 32 * C::kEpiWarp0;
        uint8_t* stg = smem + C::kStgOff + ew * 32 * stage_pitch<__nv_bfloat16>();
        __nv_bfloat16* dX = static_cast<__nv_bfloat16*>(ep.dX);
        int i = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
            const int ab = i & 1;
            const int use = i >> 1;
            const int m0 = (t / num_k) * C::kBM;
            const int k0 = (t % num_k) * BN;
            if constexpr (C::kLoraMMA) {
                // operand tables of this tile's rank-r product, tf32-rounded:
                // c*G rows m0.. and A rows k0.. (zero outside the matrices)
                uint8_t* gt = tabs;
                uint8_t* at = gt + C::kGtBytes;
                for (int e = et; e < C::kBM * C::kKL; e += 32 * C::kEpiWarps) {
                    const int rr = e / C::kKL, j = e % C::kKL;
                    const int m = m0 + rr;
                    const float g = (m < M && j < ep.r) ? g_row(ep, M, m, j) * ep.c : 0.f;
                    float hi, lo;
                    tf32_split(g, hi, lo);
                    *reinterpret_cast<float*>(gt + kmajor_tf32_offset(rr, j, C::kKL)) = hi;
                }
                for (int e = et; e < BN * C::kKL; e += 32 * C::kEpiWarps) {
                    const int cc = e / C::kKL, j = e % C::kKL;
                    const int k = k0 + cc;
                    const float a = (k < K && j < ep.r) ? a_at(ep, k, j) : 0.f;
                    float hi, lo;
                    tf32_split(a, hi, lo);
                    *reinterpret_cast<float*>(at + kmajor_tf32_offset(cc, j, C::kKL)) = hi;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&lready[ab]);
            }
            const int msub = MSUB == 2 ? sub : 0;
            const int row0 = m0 + msub * 128 + q * 32;
            const int row = row0 + lane;
            const bool row_ok = row < M;
            float gr[C::kLoraMMA ? 1 : RMAX];
            if constexpr (!C::kLoraMMA) {
#pragma unroll
                for (int j = 0; j < RMAX; ++j)
                    gr[j] = (row_ok && j < ep.r) ? g_row(ep, M, row, j) * ep.c : 0.f;
            }
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[ab], use & 1, status));
            if (!ok) break;
            tc_fence_after();
            const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + ab * C::kBufCols +
                                   msub * BN;
            const int cbeg = MSUB == 2 ? 0 : sub * (BN / C::kEpiPerQuarter);
            const int cend = MSUB == 2 ? BN : (sub + 1) * (BN / C::kEpiPerQuarter);
#pragma unroll 1
            for (int col = cbeg; col < cend; col += kEpiCols) {
                // the chains' partial sums, added in chain order
                uint32_t v[kEpiCols];
                float part[kEpiCols];
                tmem_ld16(tbase + col, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < kEpiCols; ++e) part[e] = __uint_as_float(v[e]);
#pragma unroll
                for (int ch = 1; ch < C::kKChains; ++ch) {
                    tmem_ld16(tbase + ch * C::kAccCols + col, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < kEpiCols; ++e) part[e] += __uint_as_float(v[e]);
                }
                float y[kEpiCols];
#pragma unroll
                for (int e = 0; e < kEpiCols; ++e) {
                    const int c = col + e;
                    float acc = part[e];
                    if constexpr (!C::kLoraMMA) {
                        const int k = k0 + c;
                        if (k < K)
                            for (int j = 0; j < ep.r; ++j) acc = fmaf(gr[j], a_at(ep, k, j), acc);
                    }
                    if (ep.bias && k0 + c < K) acc += __ldg(ep.bias + k0 + c);
                    y[e] = acc;
                }
                if (ep.gate && row_ok && k0 + col < K) {
                    // backward of the ReLU that produced this layer's input
                    const uint4* gp = reinterpret_cast<const uint4*>(
                        static_cast<const __nv_bfloat16*>(ep.gate) + static_cast<size_t>(row) * K + k0 + col);
                    const uint4 g0 = __ldg(gp), g1 = __ldg(gp + 1);
                    const __nv_bfloat16* gh0 = reinterpret_cast<const __nv_bfloat16*>(&g0);
                    const __nv_bfloat16* gh1 = reinterpret_cast<const __nv_bfloat16*>(&g1);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if (!(__bfloat162float(gh0[e]) > 0.f)) y[e] = 0.f;
                        if (!(__bfloat162float(gh1[e]) > 0.f)) y[8 + e] = 0.f;
                    }
                }
                store_block<__nv_bfloat16>(stg, y, lane, dX, static_cast<size_t>(K), row0, M, k0 + col,
                                           K, true);
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

template <int MSUB, int BN, int RMAX, int MODE>
cudaError_t launch_tc(const void* dY, const int8_t* Wq, const float* sw, int M, int N, int K,
                      const DxEpilogue& ep, int* status, cudaStream_t s) {
    using C = K3Cfg<MSUB, BN, RMAX>;
    auto kern = k3_dx_dequant_kernel<MSUB, BN, RMAX, MODE>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), C::kTotal);
    if (e != cudaSuccess) return e;
    // dY as [row][64-column block][64] (one 3-D box per stage) when the rows
    // split into whole blocks; otherwise one 2-D box per 64-column block
    CUtensorMap tdy;
    const int dy3d = (N % kBlkN) == 0 ? 1 : 0;
    const bool ok =
        dy3d ? make_tmap_3d_blocks(&tdy, dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, kBlkN, C::kBM,
                                   C::kBlk)
             : make_tmap_2d(&tdy, dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N,
                            static_cast<uint64_t>(N) * 2, C::kBM, kBlkN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    const int tiles = ((M + C::kBM - 1) / C::kBM) * ((K + BN - 1) / BN);
    const int grid = tiles < sm_count() ? tiles : sm_count();
    return launch_k(kern, dim3(grid), dim3(C::kThreads), C::kTotal, s, 1, tdy, dy3d, Wq, sw, M, N, K, ep,
                    status);
}

template <int RMAX, int MODE>
cudaError_t launch_tc_cfg(int cfg, const void* dY, const int8_t* Wq, const float* sw, int M, int N,
                          int K, const DxEpilogue& ep, int* status, cudaStream_t s) {
    if (cfg == 0) return launch_tc<2, 128, RMAX, MODE>(dY, Wq, sw, M, N, K, ep, status, s);
    if (cfg == 1) return launch_tc<1, 128, RMAX, MODE>(dY, Wq, sw, M, N, K, ep, status, s);
    return launch_tc<1, 64, RMAX, MODE>(dY, Wq, sw, M, N, K, ep, status, s);
}

template <int MODE>
cudaError_t launch_tc_r(int cfg, const void* dY, const int8_t* Wq, const float* sw, int M, int N,
                        int K, const DxEpilogue& ep, int* status, cudaStream_t s) {
    if (ep.r <= 4) return launch_tc_cfg<4, MODE>(cfg, dY, Wq, sw, M, N, K, ep, status, s);
    if (ep.r <= 8) return launch_tc_cfg<8, MODE>(cfg, dY, Wq, sw, M, N, K, ep, status, s);
    if (ep.r <= 16) return launch_tc_cfg<16, MODE>(cfg, dY, Wq, sw, M, N, K, ep, status, s);
    return launch_tc_cfg<64, MODE>(cfg, dY, Wq, sw, M, N, K, ep, status, s);
}

// ---------------------------------------------------------------- SIMT path
// 64 x 64 tile of dX per CTA, 256 threads (4 x 4 outputs each), n in steps of
// 16 through shared memory; the kernel tile is de-quantized on load, to fp32
// (fp32 activations) or rounded on to bf16 (bf16 activations).
constexpr int kSB = 64;
constexpr int kSN = 16;

template <typename T, int MODE>
__global__ void __launch_bounds__(256) k3_dx_simt_kernel(const T* __restrict__ dY,
                                                         const int8_t* __restrict__ Wq,
                                                         const float* __restrict__ sw, int M,
                                                         int N, int K, DxEpilogue ep) {
    __shared__ float sD[kSN][kSB + 1];  // [n][m]
    __shared__ float sW[kSN][kSB + 1];  // [n][k]
    pdl_trigger();
    pdl_wait();
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int m0 = blockIdx.y * kSB, k0 = blockIdx.x * kSB;
    float acc[4][4] = {};
    for (int n0 = 0; n0 < N; n0 += kSN) {
        for (int i = threadIdx.x; i < kSN * kSB; i += 256) {
            const int mm = i / kSN, nn = i % kSN;  // consecutive threads: consecutive n of a row
            const int m = m0 + mm, n = n0 + nn;
            sD[nn][mm] = (m < M && n < N) ? ActIO<T>::to_f(dY[static_cast<size_t>(m) * N + n]) : 0.f;
        }
        for (int i = threadIdx.x; i < kSN * kSB; i += 256) {
            const int nn = i / kSB, kk = i % kSB;
            const int n = n0 + nn, k = k0 + kk;
            float w = 0.f;
            if (n < N && k < K) {
                if constexpr (MODE == 2) {
                    const int code = reinterpret_cast<const uint8_t*>(Wq)[static_cast<size_t>(n) * K + k];
                    w = __fadd_rn(__ldg(ep.ol.par + 3), __fmul_rn(static_cast<float>(code), __ldg(ep.ol.par + 2)));
                } else {
                    int code;
                    if constexpr (MODE == 1) {
                        const int b = reinterpret_cast<const uint8_t*>(Wq)[static_cast<size_t>(n) * (K / 2) + k / 2];
                        const int nib = (k & 1) ? (b >> 4) & 0xF : b & 0xF;
                        code = nib >= 8 ? nib - 16 : nib;
                    } else {
                        code = Wq[static_cast<size_t>(n) * K + k];
                    }
                    w = __fmul_rn(static_cast<float>(code), __ldg(sw + n));
                }
                if constexpr (sizeof(T) == 2) w = __bfloat162float(__float2bfloat16_rn(w));
            }
            sW[nn][kk] = w;
        }
        if constexpr (MODE == 2) {
            // the outliers of the 16 contraction rows, columns k0 .. k0+63
            __syncthreads();
            if (threadIdx.x < kSN && n0 + static_cast<int>(threadIdx.x) < N) {
                const int n = n0 + threadIdx.x;
                const size_t b = static_cast<size_t>(n) * ep.ol.nb + (k0 >> 7);
                const int e1 = __ldg(ep.ol.start + b + 1);
                for (int e = __ldg(ep.ol.start + b); e < e1; ++e) {
                    const uint32_t v = __ldg(ep.ol.ent + e);
                    const int col = static_cast<int>(v >> 16) - (k0 & 127);
                    if (col < 0 || col >= kSB) continue;
                    float f = __half2float(__ushort_as_half(static_cast<unsigned short>(v & 0xFFFFu)));
                    if constexpr (sizeof(T) == 2) f = __bfloat162float(__float2bfloat16_rn(f));
                    sW[threadIdx.x][col] = f;
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int nn = 0; nn < kSN; ++nn) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = sD[nn][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = sW[nn][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    // G rows of this tile, summed from the column-block slices
    __shared__ float sG[kSB][65];
    for (int i = threadIdx.x; i < kSB * ep.r; i += 256) {
        const int mm = i / ep.r, jj = i % ep.r;
        sG[mm][jj] = (m0 + mm < M) ? g_row(ep, M, m0 + mm, jj) : 0.f;
    }
    __syncthreads();
    T* dX = static_cast<T*>(ep.dX);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty + 16 * i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = k0 + tx + 16 * j;
            if (k >= K) continue;
            float l = 0.f;
            for (int jj = 0; jj < ep.r; ++jj) l = fmaf(sG[ty + 16 * i][jj], a_at(ep, k, jj), l);
            const bool pass =
                !ep.gate || ActIO<T>::to_f(static_cast<const T*>(ep.gate)[static_cast<size_t>(m) * K + k]) > 0.f;
            const float b = ep.bias ? __ldg(ep.bias + k) : 0.f;
            dX[static_cast<size_t>(m) * K + k] = ActIO<T>::from_f(pass ? acc[i][j] + ep.c * l + b : 0.f);
        }
    }
}

}  // namespace

cudaError_t launch_gemm_dx(Act act, const void* dY, const int8_t* Wq, const float* sw, int M,
                           int N, int K, const DxEpilogue& ep, int* status, cudaStream_t s, bool w4) {
    const bool tc = act == kBF16 && (N % 8) == 0 && (!ep.ol.par || (K % 16) == 0);
    const int mode = ep.ol.par ? 2 : (w4 ? 1 : 0);
    if (!tc) {
        dim3 grid((K + kSB - 1) / kSB, (M + kSB - 1) / kSB);
        if (act == kBF16) {
            auto kern = mode == 2 ? k3_dx_simt_kernel<__nv_bfloat16, 2>
                                  : (mode == 1 ? k3_dx_simt_kernel<__nv_bfloat16, 1>
                                               : k3_dx_simt_kernel<__nv_bfloat16, 0>);
            return launch_k(kern, grid, dim3(256), 0, s, 1, static_cast<const __nv_bfloat16*>(dY), Wq,
                            sw, M, N, K, ep);
        }
        auto kern = mode == 2 ? k3_dx_simt_kernel<float, 2>
                              : (mode == 1 ? k3_dx_simt_kernel<float, 1> : k3_dx_simt_kernel<float, 0>);
        return launch_k(kern, grid, dim3(256), 0, s, 1, static_cast<const float*>(dY), Wq, sw, M, N, K,
                        ep);
    }
    if (mode != 2 && !ep.bias && small_m_applies(M, K, ep.r))
        return launch_gemm_dx_small(dY, Wq, sw, M, N, K, ep, status, s, w4);
    if (gemm_dx_pair_applies(M, N, K, ep.r))
        return launch_gemm_dx_pair(dY, Wq, sw, M, N, K, ep, status, s, w4);
    // tile shape: the least estimated main-loop time, i.e. waves of
    // persistent CTAs x stages per tile x the measured pace of one stage on
    // B200 (128x64 tiles: 0.88 us per 128-deep stage; 128x128: 1.30 us;
    // 256x128: 0.91 us per 64-deep stage)
    const int sms = sm_count();
    auto cost = [&](int bm, int bn, int bkn, double pace) {
        const long long tiles = static_cast<long long>((M + bm - 1) / bm) * ((K + bn - 1) / bn);
        const long long waves = (tiles + sms - 1) / sms;
        return static_cast<double>(waves) * ((N + bkn - 1) / bkn) * pace;
    };
    const double c0 = cost(256, 128, 64, 0.91), c1 = cost(128, 128, 128, 1.30),
                 c2 = cost(128, 64, 128, 0.88);
    int cfg = 2;
    if (c1 < c2 && c1 <= c0) cfg = 1;
    else if (c0 < c2 && c0 < c1) cfg = 0;
    if (mode == 2) return launch_tc_r<2>(cfg, dY, Wq, sw, M, N, K, ep, status, s);
    return w4 ? launch_tc_r<1>(cfg, dY, Wq, sw, M, N, K, ep, status, s)
              : launch_tc_r<0>(cfg, dY, Wq, sw, M, N, K, ep, status, s);
}

}  // namespace qlora
