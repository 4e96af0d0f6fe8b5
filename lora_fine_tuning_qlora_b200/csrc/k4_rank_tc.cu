// k4_rank_tc.cu -- the rank-r passes of the LoRA backward on the tensor cores
// (bf16 activations):
//
//   dY pass:  Gp[b][m,j] = sum_{n in block b} dY[m,n] B[j,n]      (G slices)
//             dB[j,n]    = c * sum_m xA[m,j] dY[m,n]
//             dbias[n]   = sum_m dY[m,n]
//   X pass:   dA[k,j]    = c * sum_m X[m,k] G[m,j]               (G = sum_b Gp[b])
//
// ("How to fine-tune the 4-bit model?" thread: the adapter's A B^T-style
// products drive the gradient; "Parameter-efficient fine-tuning of GPT-2
// with LoRA", "LoRA equation", for the shapes.)  The dY pass also runs as
// two halves, G alone and dB + dbias alone, so that a caller can put G on
// its critical path and the parameter gradients elsewhere.
//
// A CTA owns 128 columns of the activation T (dY or X) and a run of 128-row
// tiles.  Each tile arrives by TMA (one 3-D box of two 64-column blocks, or
// two 2-D boxes) with the 128-byte swizzle, and the one copy in shared
// memory is read two ways by tcgen05.mma.kind::f16 (bf16 in, fp32
// accumulate in TMEM):
//   * K-major (rows = M dimension, columns = contraction): T . Bcat^T gives
//     the tile's G rows;
//   * MN-major (columns = M dimension, rows = contraction): T^T . Vcat sums
//     over the tile's rows into a [128 columns x NV] accumulator that stays
//     in TMEM across all the CTA's tiles: dB^T and dbias, or dA.
// The fp32 factors enter as bf16 head + remainder pairs (v = hi + lo to
// about 16 significant bits; every bf16 x bf16 product is exact in fp32), so
// the sums carry about 16 significant bits of each factor, with fp32
// accumulation.  Vcat holds [xA_hi | xA_lo | 1] (the ones
// column yields dbias) or [G_hi | G_lo]; Bcat holds [B_hi | B_lo].  The head
// and remainder halves sit RP = roundup(r, 16) columns apart in TMEM, so one
// 16-column load of each gives 16 sums.
//
// Column sums: the CL <= 8 CTAs that share a column block form a cluster
// along the rows.  Each CTA owns 128/CL of the block's columns: every CTA
// stores its partials for those columns into the owner's shared memory
// (distributed shared memory) and arrives on the owner's mbarrier; the owner
// adds the CL partials in rank order, so dB, dbias and dA leave the kernel
// final and deterministic, with no cluster-wide barrier at the end.
//
// Warps: 0 TMA producer, 1 TMEM owner + MMA issuer, 2..5 operand tables and
// epilogues (warp w owns TMEM lane quarter w % 4).
#include "internal.h"
#include "ptx.cuh"

namespace qlora {

namespace {

constexpr int kTileRows = 128;
constexpr int kTileCols = 128;
constexpr int kBoxCols = 64;                         // one 128-byte swizzle row of bf16
constexpr uint32_t kBoxBytes = kTileRows * kBoxCols * 2;
constexpr uint32_t kTileBytes = 2 * kBoxBytes;
constexpr int kWorkers = 4;
constexpr int kThreads = 64 + 32 * kWorkers;
constexpr int kMaxCluster = 8;
constexpr uint32_t kTabSbo = (kTileCols / 8) * 128;  // 8-row group stride of a 128-wide table
constexpr int kMaxBulkR = 8;                         // rank limit of the bulk-copied V rows

// What one launch computes.
struct Parts {
    bool g;     // G slices from T . B^T
    bool d;     // column sums T^T . V (dB or dA), reduced over the cluster
    bool ones;  // a ones column in V (dbias)
};

struct RankTcArgs {
    const float* V;      // column sums: xA [M, r] (nsl = 1) or the nsl slices of G
    int nsl;
    const float* B;      // G: B [r, C]
    float* Gp;           // G: slices out [ceil(C/128)][M, r]
    float* out;          // column sums: dB [r, C] (with ones) or dA [C, r]
    float* dbias;        // with ones: [C] or nullptr
    int M, C, r;
    int tiles_per_cta;   // 128-row tiles per CTA
    float c;
    int vbulk;           // column sums, one V slice, r % 4 == 0, r <= kMaxBulkR, V 16-byte aligned:
                         // V's tile rows arrive by bulk copy, issued with the tile's
};

// Shared-memory and TMEM layout for rank r (same on host and device).
struct RtLayout {
    int RP, NG, NV, JP;
    uint32_t vtab, bcat, recv, bar, vraw, vslot, total;
    uint32_t tmem_cols, d_col, g_col;
    __host__ __device__ RtLayout(Parts p, int r, bool vbulk) {
        RP = (r + 15) / 16 * 16;
        NG = p.g ? 2 * RP : 0;
        NV = p.d ? 2 * RP + (p.ones ? 16 : 0) : 0;
        JP = p.d ? r + (p.ones ? 1 : 0) : 0;
        vtab = 2 * kTileBytes;
        bcat = vtab + 2 * static_cast<uint32_t>(NV) * 256;
        recv = bcat + static_cast<uint32_t>(NG) * 256;
        bar = recv + (((kTileCols + kMaxCluster) * JP * 4 + 15) / 16) * 16;
        vraw = bar + 128;  // [2][128 rows][r] fp32 with vbulk
        vslot = vbulk ? static_cast<uint32_t>(kTileRows * r * 4) : 0u;
        total = vraw + 2 * vslot;
        d_col = 0;
        g_col = static_cast<uint32_t>(NV);
        const uint32_t need = static_cast<uint32_t>(NV + 2 * NG);
        tmem_cols = 32;
        while (tmem_cols < need) tmem_cols <<= 1;
    }
};

// Byte offset of element (row, k) of a K-major bf16 operand table that is 128
// elements long in K, no swizzle: 8-row x 16-byte core matrices, K-adjacent
// ones 128 B apart (leading byte offset), 8-row groups 2048 B apart (stride
// byte offset).
__device__ __forceinline__ uint32_t ktab_off(int row, int k) {
    return static_cast<uint32_t>((row >> 3) * kTabSbo + (k >> 3) * 128 + (row & 7) * 16 +
                                 (k & 7) * 2);
}

__device__ __forceinline__ void put_split(uint8_t* tab, int row_hi, int row_lo, int k, float v) {
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    *reinterpret_cast<__nv_bfloat16*>(tab + ktab_off(row_hi, k)) = hi;
    *reinterpret_cast<__nv_bfloat16*>(tab + ktab_off(row_lo, k)) = lo;
}

template <bool kG, bool kD, bool kOnes>
__global__ void __launch_bounds__(kThreads) k4_rank_tc_kernel(const __grid_constant__ CUtensorMap tmT,
                                                              int t3d, RankTcArgs a, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const RtLayout L(Parts{kG, kD, kOnes}, a.r, kD && a.vbulk);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar);
    uint64_t* full = bars;        // [2] tile landed
    uint64_t* vready = bars + 2;  // [2] Vcat table written
    uint64_t* empty = bars + 4;   // [2] tile and table consumed by the MMAs
    uint64_t* gfull = bars + 6;   // [2] G accumulator ready
    uint64_t* gempty = bars + 8;  // [2] G accumulator read out
    uint64_t* dfull = bars + 10;  // column accumulator final
    uint64_t* rbar = bars + 11;   // every CTA of the cluster delivered this CTA's column slice
    uint64_t* vfull = bars + 12;  // [2] vbulk: the tile's V rows landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
    // recv[q][c][j]: partial of CTA q for column cbeg + c of this CTA's slice
    float* recv = reinterpret_cast<float*>(smem + L.recv);

    uint32_t CL = 1, crank = 0;
    if constexpr (kD) {
        asm("mov.u32 %0, %%cluster_nctarank;" : "=r"(CL));
        asm("mov.u32 %0, %%cluster_ctarank;" : "=r"(crank));
    }
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int cb = blockIdx.x;
    const int col0 = cb * kTileCols;
    const int mtiles = (a.M + kTileRows - 1) / kTileRows;
    const int t0 = blockIdx.y * a.tiles_per_cta;
    const int t1 = min(mtiles, t0 + a.tiles_per_cta);
    const int nt = t1 > t0 ? t1 - t0 : 0;
    // the 128 columns are split over the cluster: CTA q sums columns [q*per, q*per + per)
    const int per = (kTileCols + static_cast<int>(CL) - 1) / static_cast<int>(CL);
    const int cbeg = static_cast<int>(crank) * per;
    const int cend = min(kTileCols, cbeg + per);
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&vready[s], kWorkers);
            mbar_init(&empty[s], 1);
            mbar_init(&gfull[s], 1);
            mbar_init(&gempty[s], kWorkers);
            mbar_init(&vfull[s], 1);
        }
        mbar_init(dfull, 1);
        mbar_init(rbar, static_cast<uint32_t>(CL * (cend > cbeg ? cend - cbeg : 1)));
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, L.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // no CTA of the cluster arrives on another's barrier before all are initialised
    if constexpr (kD) cluster_arrive_relaxed();
    pdl_wait();  // nothing above read global memory

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmT);
            for (int i = 0; i < nt; ++i) {
                const int s = i & 1;
                if (i >= 2 && !mbar_wait(&empty[s], ((i >> 1) - 1) & 1, status)) break;
                uint8_t* dst = smem + s * kTileBytes;
                const int m0 = (t0 + i) * kTileRows;
                // with vbulk, the tile's rows of V (16-byte multiples: r % 4 == 0) first, on a
                // barrier of their own, so the V table is written while the tile is in flight
                if (kD && a.vbulk) {
                    const uint32_t vbytes = static_cast<uint32_t>(min(kTileRows, a.M - m0) * a.r * 4);
                    mbar_arrive_expect_tx(&vfull[s], vbytes);
                    bulk_load(smem + L.vraw + s * L.vslot, a.V + static_cast<size_t>(m0) * a.r, vbytes, &vfull[s]);
                }
                mbar_arrive_expect_tx(&full[s], kTileBytes);
                if (t3d) {  // both 64-column blocks in one box
                    tma_load_3d(dst, &tmT, &full[s], 0, m0, col0 / kBoxCols);
                } else {
                    tma_load_2d(dst, &tmT, &full[s], col0, m0);
                    tma_load_2d(dst + kBoxBytes, &tmT, &full[s], col0 + kBoxCols, m0);
                }
            }
        }
        __syncwarp();
        if constexpr (kD) cluster_wait();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t tiles = smem_u32(smem);
            const uint32_t vt = smem_u32(smem + L.vtab);
            const uint32_t bt = smem_u32(smem + L.bcat);
            const uint32_t id_g = idesc_bf16(128, kG ? L.NG : 16, false, false);
            const uint32_t id_d = idesc_bf16(128, kD ? L.NV : 16, true, false);
            bool ok = true;
            for (int i = 0; i < nt; ++i) {
                const int s = i & 1;
                // Vcat of this tile (column sums), or the Bcat table once (G alone)
                const bool need_v = kD || i == 0;
                if (!mbar_wait(&full[s], (i >> 1) & 1, status) ||
                    (need_v && !mbar_wait(&vready[s], (i >> 1) & 1, status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tb = tiles + s * kTileBytes;
                if constexpr (kG) {
                    // G rows of this tile: T (K-major) x Bcat
                    if (i >= 2 && !mbar_wait(&gempty[s], ((i >> 1) - 1) & 1, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kTileCols / 16; ++kk) {
                        const uint64_t ad = smem_desc(tb + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16,
                                                      1024, kLayoutSw128);
                        const uint64_t bd = smem_desc(bt + kk * 256, 128, kTabSbo, kLayoutNone);
                        mma_bf16(tmem + L.g_col + s * L.NG, ad, bd, id_g, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&gfull[s]);
                }
                if constexpr (kD) {
                    // column sums: T^T (MN-major, the two blocks 64 columns apart) x Vcat
#pragma unroll
                    for (int kk = 0; kk < kTileRows / 16; ++kk) {
                        const uint64_t ad = smem_desc(tb + kk * 2048, kBoxBytes, 1024, kLayoutSw128);
                        const uint64_t bd =
                            smem_desc(vt + s * L.NV * 256 + kk * 256, 128, kTabSbo, kLayoutNone);
                        mma_bf16(tmem + L.d_col, ad, bd, id_d, (i > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit(&empty[s]);
            }
            if (kD && ok) mma_commit(dfull);
        }
        __syncwarp();
        if constexpr (kD) cluster_wait();
    } else {
        // ------------------------------------------------------ tables, epilogues
        const int wq = warp & 3;
        const int rr = wq * 32 + lane;  // tile row for the tables; column for the readback
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        bool ok = true;
        if constexpr (kG) {
            // Bcat[j][n] = B[j, col0 + n] as head (rows 0..RP) and remainder (RP..2RP),
            // eight loads in flight per round
            // (loads from clamped addresses first, the zeroing of entries
            // outside B after them, so that no select waits on a single load)
            uint8_t* bt = smem + L.bcat;
            const int n = col0 + rr;
            const int nc = n < a.C ? n : a.C - 1;
            for (int j0 = 0; j0 < L.RP; j0 += 8) {
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int jc = j0 + e < a.r ? j0 + e : a.r - 1;
                    v[e] = __ldg(a.B + static_cast<size_t>(jc) * a.C + nc);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    put_split(bt, j0 + e, L.RP + j0 + e, rr, (j0 + e < a.r && n < a.C) ? v[e] : 0.f);
            }
            if constexpr (!kD) {
                // G alone: the MMAs of the first tile wait for this table on vready[0]
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&vready[0]);
            }
        }
        auto g_epilogue = [&](int i) {
            const int b = i & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&gfull[b], (i >> 1) & 1, status));
            if (!ok) return;
            tc_fence_after();
            const int m = (t0 + i) * kTileRows + rr;
            const uint32_t base = tmem + lane_base + L.g_col + b * L.NG;
            float* g = a.Gp + (static_cast<size_t>(cb) * a.M + m) * a.r;
            for (int c0 = 0; c0 < L.RP; c0 += 16) {
                uint32_t hi[16], lo[16];
                tmem_ld16(base + c0, hi);
                tmem_ld16(base + L.RP + c0, lo);
                tmem_ld_wait();
                if (m < a.M) {
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        if (c0 + e < a.r) g[c0 + e] = __uint_as_float(hi[e]) + __uint_as_float(lo[e]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&gempty[b]);
        };
        if constexpr (kG && !kD) {
            // the Bcat table is the only operand the workers write
            for (int i = 0; i < nt && ok; ++i) g_epilogue(i);
        }
        if constexpr (kD) {
            // rows of V in whole 8-float groups at 16-byte alignment
            const bool vec4 = (a.r % 8) == 0 && (reinterpret_cast<uintptr_t>(a.V) & 15) == 0;
            const int tw = threadIdx.x - 64;  // 0 .. 127
            if (a.vbulk) {
                // the parts of both V tables that no tile changes: zero rows
                // beyond r in the head and remainder halves, and the ones block
                // (a ones row, then zeros; the tile's rows past M are zero, so
                // their ones add nothing), as 16-byte chunks of 8 tile rows
                const int nconst = L.NV - 2 * a.r;
                for (int idx = tw; idx < 2 * nconst * 16; idx += 32 * kWorkers) {
                    const int b = idx / (nconst * 16), rem = idx % (nconst * 16);
                    const int jj = rem / 16, kg = rem % 16;
                    const int j = jj < L.RP - a.r ? a.r + jj : (jj < 2 * (L.RP - a.r) ? L.RP + a.r + jj - (L.RP - a.r)
                                                                                      : 2 * L.RP + jj - 2 * (L.RP - a.r));
                    const uint32_t w = (kOnes && j == 2 * L.RP) ? 0x3F803F80u : 0u;  // bf16 1.0 pairs
                    *reinterpret_cast<uint4*>(smem + L.vtab + b * L.NV * 256 + ktab_off(j, 8 * kg)) =
                        make_uint4(w, w, w, w);
                }
            }
            for (int i = 0; i < nt && ok; ++i) {
                const int s = i & 1;
                const int m = (t0 + i) * kTileRows + rr;
                ok = __all_sync(0xffffffffu,
                                i < 2 || mbar_wait(&empty[s], ((i >> 1) - 1) & 1, status));
                if (!ok) break;
                uint8_t* vt = smem + L.vtab + s * L.NV * 256;
                const bool mok = m < a.M;
                if (a.vbulk) {
                    // the tile's V rows have landed: chunk (j, kg) of the head and
                    // remainder tables from rows 8 kg .. 8 kg + 7
                    ok = __all_sync(0xffffffffu, mbar_wait(&vfull[s], (i >> 1) & 1, status));
                    if (!ok) break;
                    const float* vr = reinterpret_cast<const float*>(smem + L.vraw + s * L.vslot);
                    const int mt0 = (t0 + i) * kTileRows;
                    for (int idx = tw; idx < a.r * 16; idx += 32 * kWorkers) {
                        const int kg = idx / a.r, j = idx % a.r;
                        uint32_t hi[4], lo[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            float v2[2];
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const int row = 8 * kg + 2 * e2 + h;
                                v2[h] = mt0 + row < a.M ? vr[row * a.r + j] : 0.f;
                            }
                            const __nv_bfloat16 h0 = __float2bfloat16_rn(v2[0]), h1 = __float2bfloat16_rn(v2[1]);
                            const __nv_bfloat16 l0 = __float2bfloat16_rn(v2[0] - __bfloat162float(h0));
                            const __nv_bfloat16 l1 = __float2bfloat16_rn(v2[1] - __bfloat162float(h1));
                            hi[e2] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
                                     (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
                            lo[e2] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) |
                                     (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
                        }
                        *reinterpret_cast<uint4*>(vt + ktab_off(j, 8 * kg)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                        *reinterpret_cast<uint4*>(vt + ktab_off(L.RP + j, 8 * kg)) =
                            make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    }
                } else {
                for (int j0 = 0; j0 < L.RP; j0 += 8) {
                    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    bool vdone = false;
                    if constexpr (!kG) {
                      if (mok && j0 < a.r && vec4) {
                        vdone = true;
                        // V = the nsl slices added in ascending order: eight
                        // slices' rows in flight as 16-byte loads, then the adds
                        const float4* p4 = reinterpret_cast<const float4*>(a.V + static_cast<size_t>(m) * a.r + j0);
                        const size_t st4 = static_cast<size_t>(a.M) * a.r / 4;
                        for (int b0 = 0; b0 < a.nsl; b0 += 8) {
                            float4 lo[8], hi[8];
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const size_t b = static_cast<size_t>(b0 + u < a.nsl ? b0 + u : b0);
                                lo[u] = __ldg(p4 + b * st4);
                                hi[u] = __ldg(p4 + b * st4 + 1);
                            }
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                if (b0 + u < a.nsl) {
                                    v[0] += lo[u].x; v[1] += lo[u].y; v[2] += lo[u].z; v[3] += lo[u].w;
                                    v[4] += hi[u].x; v[5] += hi[u].y; v[6] += hi[u].z; v[7] += hi[u].w;
                                }
                            }
                        }
                      }
                    }
                    if (!vdone && mok && j0 < a.r) {
                        const int nv = min(8, a.r - j0);
                        const float* p = a.V + static_cast<size_t>(m) * a.r + j0;
                        // V = the nsl slices added in ascending order, every load issued at once
                        const size_t stride = static_cast<size_t>(a.M) * a.r;
#pragma unroll
                        for (int b = 0; b < kMaxDirectSlices; ++b)
                            if (b < a.nsl)
#pragma unroll
                                for (int e = 0; e < 8; ++e)
                                    if (e < nv) v[e] += __ldg(p + b * stride + e);
                        for (int b = kMaxDirectSlices; b < a.nsl; ++b)
                            for (int e = 0; e < nv; ++e) v[e] += __ldg(p + b * stride + e);
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) put_split(vt, j0 + e, L.RP + j0 + e, rr, v[e]);
                }
                if constexpr (kOnes) {
                    const __nv_bfloat16 one = __float2bfloat16_rn(mok ? 1.f : 0.f);
                    const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
                    *reinterpret_cast<__nv_bfloat16*>(vt + ktab_off(2 * L.RP, rr)) = one;
                    for (int j = 2 * L.RP + 1; j < L.NV; ++j)
                        *reinterpret_cast<__nv_bfloat16*>(vt + ktab_off(j, rr)) = zero;
                }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&vready[s]);
                if constexpr (kG) {
                    if (i >= 1) g_epilogue(i - 1);
                }
            }
            if constexpr (kG) {
                if (ok && nt >= 1) g_epilogue(nt - 1);
            }
            // this CTA's partial of column rr goes to the CTA that owns the column
            cluster_wait();  // every CTA of the cluster has initialised its barriers
            const int owner = rr / per;
            const uint32_t dst = dsmem_addr(recv + (static_cast<int>(crank) * per + rr - owner * per) * L.JP,
                                            static_cast<uint32_t>(owner));
            if (ok && nt > 0) ok = __all_sync(0xffffffffu, mbar_wait(dfull, 0, status));
            if (ok && nt > 0) {
                tc_fence_after();
                const uint32_t base = tmem + lane_base + L.d_col;
                for (int c0 = 0; c0 < L.RP; c0 += 16) {
                    uint32_t hi[16], lo[16];
                    tmem_ld16(base + c0, hi);
                    tmem_ld16(base + L.RP + c0, lo);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        if (c0 + e < a.r)
                            dsmem_st(dst + 4 * (c0 + e), __uint_as_float(hi[e]) + __uint_as_float(lo[e]));
                }
                if constexpr (kOnes) {
                    uint32_t ones[16];
                    tmem_ld16(base + 2 * L.RP, ones);
                    tmem_ld_wait();
                    dsmem_st(dst + 4 * a.r, __uint_as_float(ones[0]));
                }
            } else {
                for (int j = 0; j < L.JP; ++j) dsmem_st(dst + 4 * j, 0.f);
            }
            mbar_arrive_remote(dsmem_addr(rbar, static_cast<uint32_t>(owner)));
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L.tmem_cols);
    }
    if constexpr (kD) {
        // this CTA's slice of the columns: the CL partials added in rank order.
        // Once every CTA's partials have arrived nothing reads or writes this
        // CTA's shared memory from outside, so it may exit without a cluster
        // barrier.
        const int width = cend - cbeg;
        const bool got = mbar_wait_cluster(rbar, 0, status);
        if (got && width > 0) {
            for (int idx = threadIdx.x; idx < L.JP * width; idx += kThreads) {
                int j, cc;
                if constexpr (kOnes) {  // dB is [r, C]: consecutive threads take consecutive columns
                    j = idx / width;
                    cc = idx % width;
                } else {                // dA is [C, r]: consecutive threads take consecutive ranks
                    cc = idx / L.JP;
                    j = idx % L.JP;
                }
                const int col = col0 + cbeg + cc;
                if (col >= a.C) continue;
                if (kOnes && j == a.r && a.dbias == nullptr) continue;
                float sum = 0.f;
                for (int q = 0; q < static_cast<int>(CL); ++q) sum += recv[(q * per + cc) * L.JP + j];
                if constexpr (kOnes) {
                    if (j < a.r) a.out[static_cast<size_t>(j) * a.C + col] = a.c * sum;
                    else a.dbias[col] = sum;
                } else {
                    a.out[static_cast<size_t>(col) * a.r + j] = a.c * sum;
                }
            }
        }
    }
}

template <bool kG, bool kD, bool kOnes>
cudaError_t launch_tc(const void* T, RankTcArgs a, int* status, cudaStream_t s) {
    // T as [row][64-column block][64] when its rows split into whole blocks
    // (one box per tile), else one 2-D box per 64-column block
    CUtensorMap tm;
    const int t3d = (a.C % kBoxCols) == 0 ? 1 : 0;
    const bool ok =
        t3d ? make_tmap_3d_blocks(&tm, T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.M, a.C, kBoxCols,
                                  kTileRows, 2)
            : make_tmap_2d(&tm, T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.M, a.C,
                           static_cast<uint64_t>(a.C) * 2, kTileRows, kBoxCols,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    a.vbulk = (kD && a.nsl == 1 && a.r % 4 == 0 && a.r <= kMaxBulkR &&
               (reinterpret_cast<uintptr_t>(a.V) & 15) == 0)
                  ? 1
                  : 0;
    const RtLayout L(Parts{kG, kD, kOnes}, a.r, kD && a.vbulk);
    if (L.tmem_cols > 512) return cudaErrorInvalidValue;  // never reached for r <= 64
    const size_t smem = L.total + 1024;
    auto kern = k4_rank_tc_kernel<kG, kD, kOnes>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int mtiles = (a.M + kTileRows - 1) / kTileRows;
    int cl = 1;
    int rows_grid;
    if (kD) {
        // rows split over a cluster of CL CTAs, every CTA at least one tile;
        // CTAs too large for two per SM take clusters of at most 4 (clusters
        // of 8 single-CTA SMs do not all fit one wave of the GPCs)
        const int max_cl = smem > 110 * 1024 ? 4 : kMaxCluster;
        a.tiles_per_cta = (mtiles + max_cl - 1) / max_cl;
        // a caller's minimum rows per CTA (fewer CTAs that stay longer)
        const int want = (rank_pass_rows() + kTileRows - 1) / kTileRows;
        if (want > a.tiles_per_cta) a.tiles_per_cta = want;
        cl = (mtiles + a.tiles_per_cta - 1) / a.tiles_per_cta;
        rows_grid = cl;
    } else {
        // G alone needs no reduction over rows: one 128-row tile per CTA,
        // unless that makes more than a few waves of CTAs
        const long long cbs = (a.C + kTileCols - 1) / kTileCols;
        a.tiles_per_cta = 1;
        while (cbs * ((mtiles + a.tiles_per_cta - 1) / a.tiles_per_cta) > 4LL * sm_count())
            a.tiles_per_cta *= 2;
        rows_grid = (mtiles + a.tiles_per_cta - 1) / a.tiles_per_cta;
    }
    const dim3 grid((a.C + kTileCols - 1) / kTileCols, rows_grid);
    return launch_k(kern, grid, dim3(kThreads), smem, s, cl, tm, t3d, a, status);
}

}  // namespace

int rank_tc_col_blocks(int C) { return (C + kTileCols - 1) / kTileCols; }

cudaError_t launch_rank_dy_tc(const void* dY, const float* B, const float* xA, int M, int N, int r,
                              float c, float* Gp, float* dB, float* dbias, int* status,
                              cudaStream_t s) {
    RankTcArgs a{};
    a.V = xA;
    a.nsl = 1;
    a.B = B;
    a.Gp = Gp;
    a.out = dB;
    a.dbias = dbias;
    a.M = M;
    a.C = N;
    a.r = r;
    a.c = c;
    if (Gp && dB) return launch_tc<true, true, true>(dY, a, status, s);
    if (Gp) return launch_tc<true, false, false>(dY, a, status, s);
    if (dB) return launch_tc<false, true, true>(dY, a, status, s);
    return cudaSuccess;
}

cudaError_t launch_rank_x_tc(const void* X, const float* G, int nsl, int M, int K, int r, float c,
                             float* dA, int* status, cudaStream_t s) {
    RankTcArgs a{};
    a.V = G;
    a.nsl = nsl;
    a.out = dA;
    a.M = M;
    a.C = K;
    a.r = r;
    a.c = c;
    return launch_tc<false, true, false>(X, a, status, s);
}

}  // namespace qlora
