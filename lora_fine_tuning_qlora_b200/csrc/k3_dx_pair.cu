// k3_dx_pair.cu -- the input gradient of the int8-LoRA Dense layer on CTA
// pairs, for large M:
//
//   dX[m,k] = sum_n dY[m,n] * bf16(Wq[n,k] * sw[n]) + c * sum_j G[m,j] A[k,j]
//
// The frozen int8 kernel is de-quantized tile by tile in shared memory right
// before the tensor-core product ("How to fine-tune the 4-bit model?"
// thread: decompress the quantized weights in place, then feed the matrix
// unit).  Here a cluster of two CTAs computes a 256 x 256 tile of dX with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16): CTA r of the pair
// loads dY rows [128 r, 128 r + 128) of the tile (TMA, K-major, 128-byte
// swizzle), de-quantizes kernel columns [128 r, 128 r + 128) of the tile
// (MN-major, 128-byte swizzle), and holds its 128 rows x 256 columns of the
// fp32 accumulator in its TMEM.  Against one CTA per 256 x 128 tile this
// halves the shared-memory bytes the tensor cores read per flop and issues a
// quarter of the MMA instructions, with the same de-quantization per flop.
//
// Warps per CTA: 0 TMA producer; 1 TMEM owner (pair allocation) and, in
// CTA 0, the MMA issuer; 2..11 de-quantize (five groups of two, one per
// stage of the five-stage ring); 12..15 epilogue.
// Barriers: full[s] (CTA 0) completes when both CTAs' dY boxes of stage s
// have landed (the second CTA's box signals it across the pair); wready[s]
// (CTA 0) takes an arrival from every warp of the de-quantize group that
// converted stage s, in both CTAs; the
// MMAs' commits arrive on empty[s] and tfull[b] in both CTAs; tempty[b]
// (CTA 0) takes an arrival from every epilogue warp of both CTAs.  The
// arrivals across the pair use CTA-scope release (the de-quantized tile stays
// in the writer's own shared memory, made visible to the tensor cores by a
// proxy fence): a cluster-scope release would wait for the de-quantize
// warps' prefetch loads in flight at every stage.  Every wait is bounded.
// The rank-r term c G A^T is added by the epilogue on CUDA cores (fp32 FMAs)
// from the G rows and a table of the tile's A rows.
#include "internal.h"
#include "ptx.cuh"
#include "tile_epilogue.cuh"
#include "dx_common.cuh"

namespace qlora {

namespace {

constexpr int kPM = 128;             // dX rows per CTA (256 per pair)
constexpr int kPN = 256;             // dX columns per pair tile (128 de-quantized per CTA)
constexpr int kPK = 64;              // contraction (n) per stage: one 64-column dY block
constexpr int kDqW = 10;             // de-quantize warps
constexpr int kDqGroups = 5;         // stage groups of de-quantize warps (two warps each)
constexpr int kDqWPG = kDqW / kDqGroups;
constexpr int kEpiW = 4;             // epilogue warps: one per TMEM lane quarter
constexpr int kDqWarp0 = 2;
constexpr int kEpiWarp0 = kDqWarp0 + kDqW;
constexpr int kPThreads = 32 * (kEpiWarp0 + kEpiW);
constexpr int kPSmemLimit = 232448;
constexpr uint32_t kPLbo = (kPK / 8) * 1024;  // MN-block stride of the de-quantized half tile

template <int RP>
struct PairCfg {
    static constexpr int kABytes = kPM * kPK * 2;         // dY rows of this CTA: 16 KB
    static constexpr int kWBytes = kPK * (kPN / 2) * 2;   // de-quantized half tile: 16 KB
    static constexpr int kStageBytes = kABytes + kWBytes;
    static constexpr int kStgBytes = kEpiW * 32 * stage_pitch<__nv_bfloat16>();
    static constexpr int kATabBytes = kPN * (RP + 1) * 4;  // A rows (+ bias) of the tile's 256 columns
    static constexpr int kFixed = kStgBytes + kATabBytes + 512 + 1024;
    static constexpr int kStagesFit = (kPSmemLimit - kFixed) / kStageBytes;
    // a multiple of the stage groups.  A group may start stage g only when the
    // MMAs of stage g - STAGES are done, so the other STAGES - 1 stages'
    // MMAs are the window its load-convert-store-signal chain must fit in:
    // five stages with five groups ran 462 us against 484 for four with
    // four at 16384 x 4096 x 4096; six groups (576 threads) spill
    static constexpr int STAGES = 5;
    static_assert(kStagesFit >= STAGES, "shared memory budget");
    static constexpr int kStgOff = STAGES * kStageBytes;
    static constexpr int kATabOff = kStgOff + kStgBytes;
    static constexpr int kBarOff = kATabOff + kATabBytes;
    static constexpr int kTotal = kBarOff + 512 + 1024;
    static constexpr uint32_t kAccCols = kPN;             // one fp32 accumulator: 256 columns
    static constexpr uint32_t kTmemCols = 2 * kAccCols;   // two buffers: all 512 columns
};

// MODE: 0 int8 codes with a scale per contraction row; 1 packed int4 codes;
// 2 outlier-compensated uint8 affine codes (ep.ol) with their fp16 outliers
// written over the de-quantized tile.
template <int RP, int MODE>
__global__ void __launch_bounds__(kPThreads, 1)
    k3_dx_pair_kernel(const __grid_constant__ CUtensorMap tmDY, const int8_t* __restrict__ Wq,
                      const float* __restrict__ sw, int M, int N, int K, DxEpilogue ep,
                      int* status) {
    using C = PairCfg<RP>;
    constexpr int S = C::STAGES;
    constexpr bool W4 = MODE == 1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);  // [S] (CTA 0)
    uint64_t* wready = full + S;                                      // [S] (CTA 0)
    uint64_t* empty = wready + S;                                     // [S]
    uint64_t* tfull = empty + S;                                      // [2]
    uint64_t* tempty = tfull + 2;                                     // [2] (CTA 0)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    float* sAt = reinterpret_cast<float*>(smem + C::kATabOff);        // [256][RP]
    float* sBias = sAt + kPN * RP;                                     // [256]

    const uint32_t rank = cluster_ctarank();
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int pair = static_cast<int>(blockIdx.x) / 2;
    const int npairs = static_cast<int>(gridDim.x) / 2;
    const int num_kt = (K + kPN - 1) / kPN;
    const int tiles = ((M + 2 * kPM - 1) / (2 * kPM)) * num_kt;
    const int nkb = (N + kPK - 1) / kPK;
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&wready[s], 2 * kDqWPG);  // one stage group of each CTA
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 2 * kEpiW);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // neither CTA signals the other's barriers before both have initialised them
    cluster_arrive();
    cluster_wait();
    pdl_wait();  // nothing above touched global memory

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmDY);
            const uint32_t full0 = dsmem_addr(full, 0);  // CTA 0's full[0]
            int g = 0;
            bool ok = true;
            for (int t = pair; t < tiles && ok; t += npairs) {
                const int m0 = (t / num_kt) * 2 * kPM + static_cast<int>(rank) * kPM;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % S;
                    if (g >= S && !mbar_wait(&empty[s], ((g / S) - 1) & 1, status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + s * C::kStageBytes;
                    if (rank == 0) {
                        mbar_arrive_expect_tx(&full[s], 2 * C::kABytes);
                        tma_load_3d(sa, &tmDY, &full[s], 0, m0, kb);
                    } else {
                        tma_load_3d_pair(sa, &tmDY, full0 + 8u * static_cast<uint32_t>(s), 0, m0, kb);
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer (CTA 0)
        if (rank == 0 && lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(2 * kPM, kPN, false, true);
            int g = 0, i = 0;
            bool ok = true;
            for (int t = pair; t < tiles && ok; t += npairs, ++i) {
                const int ab = i & 1;
                const int use = i >> 1;
                if (use > 0 && !mbar_wait(&tempty[ab], (use - 1) & 1, status)) break;
                tc_fence_after();
                const uint32_t dacc = tmem + ab * C::kAccCols;
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
                    for (int kk = 0; kk < kPK / 16; ++kk) {
                        const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024, kLayoutSw128);
                        const uint64_t bd = smem_desc(w_base + kk * 2048, kPLbo, 1024, kLayoutSw128);
                        mma_bf16_pair(dacc, ad, bd, idesc, (kb != 0 || kk != 0) ? 1u : 0u);
                    }
                    mma_commit_pair(&empty[s], 0x3);
                }
                if (ok) mma_commit_pair(&tfull[ab], 0x3);
            }
        }
        __syncwarp();
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------ de-quantize
        // The warps form kDqGroups groups; group q converts the stages
        // g = q, q + kDqGroups, ... (all of a stage's 64 x 128 codes), so a
        // warp has kDqGroups stage-times for each of its stages: the pace is
        // set by the warps' throughput, not by the latency of one stage's
        // load-convert-store-signal chain.  The codes and row scales of a
        // group's next kDqDepth stages are held in registers (loaded that
        // many group stages ahead); a chunk outside the matrices is zeroed
        // through its scale.  The stage and tile cursors advance without
        // divisions.
        const int dw = warp - kDqWarp0;
        const int grp = dw / kDqWPG;
        const int gw = dw % kDqWPG;
        constexpr int kCodes = W4 ? 32 : 16;  // codes per 16-byte chunk
        constexpr int kHalf = kPN / 2;
        constexpr int kChunksPerRow = kHalf / kCodes;
        constexpr int kChunks = kPK * kChunksPerRow;
        constexpr int kPerLane = kChunks / (32 * kDqWPG);
        static_assert(kChunks % (32 * kDqWPG) == 0, "chunks per stage");
        constexpr int P = S / kDqGroups;  // register ring of a group
        static_assert(S % kDqGroups == 0, "stages per group");
        const size_t row_bytes = W4 ? static_cast<size_t>(K) / 2 : static_cast<size_t>(K);
        const int my_tiles = pair < tiles ? (tiles - 1 - pair) / npairs + 1 : 0;
        const int total_kb = my_tiles * nkb;
        const uint32_t wready0 = dsmem_addr(wready, 0);
        // fetch cursor: stage g = grp + kDqGroups * j -> (tile ft of this pair, block fkb)
        int fj = 0, ft = 0, fkb = grp;
        while (fkb >= nkb) { fkb -= nkb; ++ft; }
        int fk0 = ((pair + ft * npairs) % num_kt) * kPN + static_cast<int>(rank) * kHalf;
        uint4 qr[P][kPerLane];
        float sr[P][kPerLane];
        uint32_t inb[P];
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
                const int c = gw * 32 + lane + i * 32 * kDqWPG;
                int cr, cc;
                chunk_rc<kChunksPerRow>(c, cr, cc);
                const int n = fkb * kPK + cr;
                const int k = fk0 + cc * kCodes;
                if (live_g && n < N && k < K) in_bits |= 1u << i;
                const int nc = n < N ? n : N - 1;
                const int kc = k < K ? k : K - kCodes;
                q[i] = __ldg(reinterpret_cast<const uint4*>(Wq + static_cast<size_t>(nc) * row_bytes +
                                                            (W4 ? kc / 2 : kc)));
                sc[i] = MODE == 2 ? 1.f : __ldg(sw + nc);
            }
            // advance to the group's next stage
            ++fj;
            fkb += kDqGroups;
            bool moved = false;
            while (fkb >= nkb) {
                fkb -= nkb;
                ++ft;
                moved = true;
            }
            if (moved) fk0 = ((pair + ft * npairs) % num_kt) * kPN + static_cast<int>(rank) * kHalf;
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
                    const int c = gw * 32 + lane + i * 32 * kDqWPG;
                    int nr, kc;
                    chunk_rc<kChunksPerRow>(c, nr, kc);
                    const float scale = (inb[v] >> i) & 1u ? sr[v][i] : 0.f;
                    const int mn = kc * kCodes;
                    uint32_t o[8];
                    if constexpr (W4) {
                        uint4 lo, hi;
                        unpack_int4x32(qr[v][i], lo, hi);
                        dequant16(lo, scale, o);
                        *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn, nr, kPLbo)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn + 8, nr, kPLbo)) =
                            make_uint4(o[4], o[5], o[6], o[7]);
                        dequant16(hi, scale, o);
                        *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn + 16, nr, kPLbo)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn + 24, nr, kPLbo)) =
                            make_uint4(o[4], o[5], o[6], o[7]);
                    } else {
                        if constexpr (MODE == 2) {
                            // outside the matrices: zero through the affine parameters
                            const bool in = (inb[v] >> i) & 1u;
                            dequant16_affine(qr[v][i], in ? ascale : 0.f, in ? abias : 0.f, o);
                        } else {
                            dequant16(qr[v][i], scale, o);
                        }
                        *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn, nr, kPLbo)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<uint4*>(wt + mn_sw128_offset(mn + 8, nr, kPLbo)) =
                            make_uint4(o[4], o[5], o[6], o[7]);
                    }
                }
                if constexpr (MODE == 2) {
                    // The warp wrote whole tile rows nr = kRW gw + (c % 32) /
                    // kChunksPerRow + kRW kDqWPG i (kRW rows per 32 chunks);
                    // its lanes now write those rows' outliers.
                    constexpr int kRW = 32 / kChunksPerRow;
                    __syncwarp();
                    const int t = pair + (g / nkb) * npairs;
                    const int c0 = (t % num_kt) * kPN + static_cast<int>(rank) * kHalf;
                    for (int idx = lane; idx < kPerLane * kRW; idx += 32) {
                        const int nr = gw * kRW + idx % kRW + kRW * kDqWPG * (idx / kRW);
                        const int n = (g % nkb) * kPK + nr;
                        if (n < N && c0 < K) patch_outliers(ep.ol, n, c0, kHalf, wt, nr, kPLbo);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (rank == 0) mbar_arrive(&wready[u]);
                    else mbar_arrive_remote_cta(wready0 + 8u * static_cast<uint32_t>(u));
                }
                fetch(qr[v], sr[v], inb[v]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int ew = warp - kEpiWarp0;     // 0 .. 3
        const int q = warp & 3;              // TMEM lane quarter of this warp
        const int et = threadIdx.x - 32 * kEpiWarp0;
        uint8_t* stg = smem + C::kStgOff + ew * 32 * stage_pitch<__nv_bfloat16>();
        __nv_bfloat16* dX = static_cast<__nv_bfloat16*>(ep.dX);
        const uint32_t tempty0 = dsmem_addr(tempty, 0);
        int i = 0;
        for (int t = pair; t < tiles; t += npairs, ++i) {
            const int ab = i & 1;
            const int use = i >> 1;
            const int m0 = (t / num_kt) * 2 * kPM + static_cast<int>(rank) * kPM;
            const int k0 = (t % num_kt) * kPN;
            // A rows of the tile's columns (the last tile's reads are done)
            named_bar_sync(1, 32 * kEpiW);
            for (int col = et; col < kPN; col += 32 * kEpiW)
                sBias[col] = (ep.bias && k0 + col < K) ? __ldg(ep.bias + k0 + col) : 0.f;
            for (int e = et; e < kPN * RP; e += 32 * kEpiW) {
                const int col = e / RP, j = e % RP;
                const int k = k0 + col;
                sAt[e] = (k < K && j < ep.r) ? a_at(ep, k, j) : 0.f;
            }
            named_bar_sync(1, 32 * kEpiW);
            const int row0 = m0 + q * 32;
            const int row = row0 + lane;
            const bool row_ok = row < M;
            float gr[RP];
#pragma unroll
            for (int j = 0; j < RP; ++j) gr[j] = (row_ok && j < ep.r) ? g_row(ep, M, row, j) * ep.c : 0.f;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[ab], use & 1, status));
            if (!ok) break;
            tc_fence_after();
            const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + ab * C::kAccCols;
#pragma unroll 1
            for (int col = 0; col < kPN; col += kEpiCols) {
                uint32_t v[kEpiCols];
                tmem_ld16(tbase + col, v);
                tmem_ld_wait();
                float y[kEpiCols];
#pragma unroll
                for (int e = 0; e < kEpiCols; ++e) {
                    const float4* a4 = reinterpret_cast<const float4*>(sAt + (col + e) * RP);
                    float acc = __uint_as_float(v[e]) + sBias[col + e];
#pragma unroll
                    for (int j4 = 0; j4 < RP / 4; ++j4) {
                        const float4 a = a4[j4];
                        acc = fmaf(gr[4 * j4 + 0], a.x, acc);
                        acc = fmaf(gr[4 * j4 + 1], a.y, acc);
                        acc = fmaf(gr[4 * j4 + 2], a.z, acc);
                        acc = fmaf(gr[4 * j4 + 3], a.w, acc);
                    }
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
                store_block<__nv_bfloat16>(stg, y, lane, dX, static_cast<size_t>(K), row0, M, k0 + col, K,
                                           true);
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
        tmem_dealloc_pair(tmem, C::kTmemCols);
    }
}

template <int RP, int MODE>
cudaError_t launch_pair_t(const void* dY, const int8_t* Wq, const float* sw, int M, int N, int K,
                          const DxEpilogue& ep, int* status, cudaStream_t s) {
    using C = PairCfg<RP>;
    auto kern = k3_dx_pair_kernel<RP, MODE>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), C::kTotal);
    if (e != cudaSuccess) return e;
    // dY as [row][64-column block][64]: one box of 128 rows x one block per stage
    CUtensorMap tdy;
    if (!make_tmap_3d_blocks(&tdy, dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, kPK, kPM, 1))
        return cudaErrorInvalidValue;
    const int tiles = ((M + 2 * kPM - 1) / (2 * kPM)) * ((K + kPN - 1) / kPN);
    const int pairs = tiles < sm_count() / 2 ? tiles : sm_count() / 2;
    // at the greatest priority: a rank pass issued beside it on another stream
    // takes only the SMs its pairs leave (its last partial wave of tiles)
    return launch_kx_urgent(kern, dim3(2 * pairs), dim3(kPThreads), C::kTotal, s, 2, tdy, Wq, sw, M, N, K,
                     ep, status);
}

}  // namespace

bool gemm_dx_pair_applies(int M, int N, int K, int r) {
    if (N % kPK != 0 || K % 16 != 0 || r > 16) return false;
    const int tiles = ((M + 2 * kPM - 1) / (2 * kPM)) * ((K + kPN - 1) / kPN);
    // from half a wave of pairs: at 1024 tokens of the 4096^2 layer (64 pair
    // tiles) the pairs ran 48.5 us against 58.7 for the single-CTA kernel's
    // 1.7 waves of 128 x 128 tiles, and on the GPT-2 projections (48 tiles)
    // 34 against 38 us (qkv), 40 against 47 (mlp up), the outlier-compensated
    // layers' steps 4-11 us faster
    return tiles >= sm_count() / 4;
}

template <int MODE>
cudaError_t launch_pair_mode(const void* dY, const int8_t* Wq, const float* sw, int M, int N,
                             int K, const DxEpilogue& ep, int* status, cudaStream_t s) {
    if (ep.r <= 4) return launch_pair_t<4, MODE>(dY, Wq, sw, M, N, K, ep, status, s);
    if (ep.r <= 8) return launch_pair_t<8, MODE>(dY, Wq, sw, M, N, K, ep, status, s);
    return launch_pair_t<16, MODE>(dY, Wq, sw, M, N, K, ep, status, s);
}

cudaError_t launch_gemm_dx_pair(const void* dY, const int8_t* Wq, const float* sw, int M, int N,
                                int K, const DxEpilogue& ep, int* status, cudaStream_t s, bool w4) {
    if (ep.ol.par) return launch_pair_mode<2>(dY, Wq, sw, M, N, K, ep, status, s);
    return w4 ? launch_pair_mode<1>(dY, Wq, sw, M, N, K, ep, status, s)
              : launch_pair_mode<0>(dY, Wq, sw, M, N, K, ep, status, s);
}

}  // namespace qlora
