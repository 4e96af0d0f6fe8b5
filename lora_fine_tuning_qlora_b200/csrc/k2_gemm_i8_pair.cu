// k2_gemm_i8_pair.cu -- the forward int8 GEMM of the int8-LoRA Dense layer on
// CTA pairs, for large layers:
//
//   acc[m,n] = sum_k Xq[m,k] Wq[n,k]                               (int32)
//   Y[m,n]   = acc * sx[m] * sw[n] + bias[n] + sum_j (c xA[m,j]) B[j,n]
//
// ("Introduce QLoRA-like technique", Results: int8 Dense needs a hardware
// int8 matmul; "Parameter-efficient fine-tuning of GPT-2 with LoRA", "LoRA
// equation" for the low-rank term.)  A cluster of two CTAs computes a
// 256 x 256 tile of Y with tcgen05.mma.cta_group::2.kind::i8 (M = 256,
// N = 256, K = 32): CTA r loads Xq rows [128 r, 128 r + 128) and Wq rows
// (output channels) [128 r, 128 r + 128) of the tile, 128 k per stage (TMA,
// K-major, 128-byte swizzle), and holds its 128 rows x 256 columns of the
// int32 accumulator in TMEM.  One MMA instruction does four times the work
// of the single-CTA kernel's 128 x 128 x 32 step, whose issue rate bounds
// that kernel at about 70% of the int8 peak.
//
// Warps per CTA: 0 TMA producer; 1 TMEM owner (pair allocation) and, in
// CTA 0, the MMA issuer; 2..5 epilogue (one per TMEM lane quarter).
// Barriers: full[s] (CTA 0) completes when all four boxes of stage s (Xq and
// Wq of both CTAs) have landed; the MMAs' commits arrive on empty[s] and
// tfull[b] in both CTAs; tempty[b] (CTA 0) takes an arrival from every
// epilogue warp of both CTAs (CTA-scope release).  Every wait is bounded.
// The epilogue applies both scales, the bias and the rank-r term on CUDA
// cores (fp32), from per-tile tables of sw, bias and B.
//
// W4 (packed int4 codes Wp [N, K/2]): each CTA's TMA brings its stage's
// packed tile ([128 rows][64 bytes], no swizzle) onto a barrier of its own
// (pfull), and warps 6..15 expand it into the int8 tile the TMA would have
// written (16-byte chunk c of row n at c ^ (n % 8)) and arrive on CTA 0's
// wready (CTA-scope release: the tile stays in the writer's shared memory,
// published to the tensor cores by a proxy fence); the MMA waits for both
// CTAs' tiles.  The expansion warps form five groups of two, one per stage of
// the five-stage ring (group q takes stages q, q + 5, ...), so a group's
// wait-expand-signal chain has the other stages' MMAs to hide in (all warps
// on every stage: 278 us at 16384 x 4096 x 4096; the groups: 231).
#include "internal.h"
#include "ptx.cuh"
#include "tile_epilogue.cuh"

namespace qlora {

namespace {

constexpr int kQM = 128;             // rows per CTA (256 per pair)
constexpr int kQN = 256;             // output columns per pair tile (128 of Wq per CTA)
constexpr int kQK = 128;             // int8 k per stage: one 128-byte swizzle row
constexpr int kQEpi = 4;             // epilogue warps
constexpr int kQUGroups = 5;         // W4: stage groups of expansion warps (one per stage of the ring)
constexpr int kQUWPG = 2;            // W4: warps per stage group
constexpr int kQUnpack = kQUGroups * kQUWPG;  // W4: warps that expand the packed codes
template <bool W4>
__host__ __device__ constexpr int q_threads() { return 32 * (2 + kQEpi + (W4 ? kQUnpack : 0)); }
constexpr int kQSmemLimit = 232448;

template <int RP, bool W4>
struct PairFwdCfg {
    static constexpr int kABytes = kQM * kQK;             // Xq rows of this CTA: 16 KB
    static constexpr int kBBytes = (kQN / 2) * kQK;       // Wq rows of this CTA: 16 KB
    static constexpr int kPBytes = W4 ? (kQN / 2) * kQK / 2 : 0;  // packed codes: 8 KB
    static constexpr int kStageBytes = kABytes + kBBytes + kPBytes;
    static constexpr int kStgBytes = kQEpi * 32 * stage_pitch<__nv_bfloat16>();
    static constexpr int kTabBytes = kQN * (RP + 2) * 4;  // B rows, sw, bias of the tile's columns
    static constexpr int kFixed = kStgBytes + kTabBytes + 512 + 1024;
    static constexpr int kStagesFit = (kQSmemLimit - kFixed) / kStageBytes;
    static constexpr int STAGES = kStagesFit > 6 ? 6 : kStagesFit;
    static_assert(STAGES >= 3, "shared memory budget");
    static_assert(!W4 || STAGES % kQUGroups == 0, "W4: stages per expansion group");
    static constexpr int kStgOff = STAGES * kStageBytes;
    static constexpr int kTabOff = kStgOff + kStgBytes;
    static constexpr int kBarOff = kTabOff + kTabBytes;
    static constexpr int kTotal = kBarOff + 512 + 1024;
    static_assert(6 * 8 * 4 + 8 * 4 <= 512, "barrier area");
    static constexpr uint32_t kAccCols = kQN;             // int32 accumulator: 256 columns
    static constexpr uint32_t kTmemCols = 2 * kAccCols;   // two buffers: all 512 columns
};

template <int RP, bool W4>
__global__ void __launch_bounds__(q_threads<W4>(), 1)
    k2_gemm_i8_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB, int M, int N, int K,
                           FwdEpilogue ep, int* status) {
    using C = PairFwdCfg<RP, W4>;
    constexpr int S = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);  // [S] (CTA 0)
    uint64_t* empty = full + S;                                       // [S]
    uint64_t* tfull = empty + S;                                      // [2]
    uint64_t* tempty = tfull + 2;                                     // [2] (CTA 0)
    uint64_t* pfull = tempty + 2;                                     // [S] W4: packed tile landed
    uint64_t* wready = pfull + S;                                     // [S] W4 (CTA 0): both tiles expanded
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wready + S);
    float* sB = reinterpret_cast<float*>(smem + C::kTabOff);          // [256][RP]
    float* sSw = sB + kQN * RP;                                        // [256]
    float* sBias = sSw + kQN;                                          // [256]

    const uint32_t rank = cluster_ctarank();
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int pair = static_cast<int>(blockIdx.x) / 2;
    const int npairs = static_cast<int>(gridDim.x) / 2;
    const int num_nt = (N + kQN - 1) / kQN;
    const int tiles = ((M + 2 * kQM - 1) / (2 * kQM)) * num_nt;
    const int nkb = (K + kQK - 1) / kQK;
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 2 * kQEpi);
        }
        if constexpr (W4)
            for (int s = 0; s < S; ++s) {
                mbar_init(&pfull[s], 1);
                mbar_init(&wready[s], 2 * kQUWPG);
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
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            const uint32_t full0 = dsmem_addr(full, 0);  // CTA 0's full[0]
            int g = 0;
            bool ok = true;
            for (int t = pair; t < tiles && ok; t += npairs) {
                const int m0 = (t / num_nt) * 2 * kQM + static_cast<int>(rank) * kQM;
                const int n0 = (t % num_nt) * kQN + static_cast<int>(rank) * (kQN / 2);
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % S;
                    if (g >= S && !mbar_wait(&empty[s], ((g / S) - 1) & 1, status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + s * C::kStageBytes;
                    if constexpr (W4) {
                        // Xq of both CTAs on CTA 0's full; each CTA's packed codes on its own pfull
                        if (rank == 0) {
                            mbar_arrive_expect_tx(&full[s], 2 * C::kABytes);
                            tma_load_2d(sa, &tmA, &full[s], kb * kQK, m0);
                        } else {
                            tma_load_2d_pair(sa, &tmA, full0 + 8u * static_cast<uint32_t>(s), kb * kQK, m0);
                        }
                        mbar_arrive_expect_tx(&pfull[s], C::kPBytes);
                        tma_load_2d(sa + C::kABytes + C::kBBytes, &tmB, &pfull[s], kb * (kQK / 2), n0);
                    } else if (rank == 0) {
                        mbar_arrive_expect_tx(&full[s], 2 * C::kStageBytes);
                        tma_load_2d(sa, &tmA, &full[s], kb * kQK, m0);
                        tma_load_2d(sa + C::kABytes, &tmB, &full[s], kb * kQK, n0);
                    } else {
                        const uint32_t fb = full0 + 8u * static_cast<uint32_t>(s);
                        tma_load_2d_pair(sa, &tmA, fb, kb * kQK, m0);
                        tma_load_2d_pair(sa + C::kABytes, &tmB, fb, kb * kQK, n0);
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer (CTA 0)
        if (rank == 0 && lane == 0) {
            constexpr uint32_t idesc = idesc_i8(2 * kQM, kQN);
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
                        (W4 && !mbar_wait(&wready[s], (g / S) & 1, status))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + s * C::kStageBytes);
                    const uint32_t b_base = a_base + C::kABytes;
#pragma unroll
                    for (int kk = 0; kk < kQK / 32; ++kk) {
                        const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024, kLayoutSw128);
                        const uint64_t bd = smem_desc(b_base + kk * 32, 16, 1024, kLayoutSw128);
                        mma_i8_pair(dacc, ad, bd, idesc, (kb != 0 || kk != 0) ? 1u : 0u);
                    }
                    mma_commit_pair(&empty[s], 0x3);
                }
                if (ok) mma_commit_pair(&tfull[ab], 0x3);
            }
        }
        __syncwarp();
    } else if (W4 && warp >= 2 + kQEpi) {
        // ------------------------------------------------------ int4 expand (W4)
        const int ew = warp - (2 + kQEpi);            // 0 .. kQUnpack - 1
        const int grp = ew / kQUWPG;                   // this warp's stage group
        const int tg = (ew % kQUWPG) * 32 + lane;      // 0 .. 32 kQUWPG - 1
        const uint32_t wready0 = dsmem_addr(wready, 0);
        int g = 0;
        bool ok = true;
        for (int tt = pair; tt < tiles && ok; tt += npairs) {
            for (int kb = 0; kb < nkb; ++kb, ++g) {
                const int s = g % S;
                if (g % kQUGroups != grp) continue;  // another group's stage
                if (!__all_sync(0xffffffffu, mbar_wait(&pfull[s], (g / S) & 1, status))) {
                    ok = false;
                    break;
                }
                uint8_t* wb = smem + s * C::kStageBytes + C::kABytes;
                const uint8_t* pk = wb + C::kBBytes;
                // 512 chunks of 32 codes (128 rows x 4) over the group's threads
                constexpr int kPer = 512 / (32 * kQUWPG);
                uint4 raw[kPer];
#pragma unroll
                for (int u = 0; u < kPer; ++u) {
                    const int e = tg + u * 32 * kQUWPG;
                    raw[u] = *reinterpret_cast<const uint4*>(pk + (e >> 2) * 64 + (e & 3) * 16);
                }
#pragma unroll
                for (int u = 0; u < kPer; ++u) {
                    const int e = tg + u * 32 * kQUWPG;
                    const int n = e >> 2, p = e & 3;
                    uint4 lo, hi;
                    unpack_int4x32(raw[u], lo, hi);
                    uint8_t* row = wb + n * kQK;
                    *reinterpret_cast<uint4*>(row + (((2 * p) ^ (n & 7)) << 4)) = lo;
                    *reinterpret_cast<uint4*>(row + (((2 * p + 1) ^ (n & 7)) << 4)) = hi;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (rank == 0) mbar_arrive(&wready[s]);
                    else mbar_arrive_remote_cta(wready0 + 8u * static_cast<uint32_t>(s));
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int ew = warp - 2;             // 0 .. 3
        const int q = warp & 3;              // TMEM lane quarter of this warp
        const int et = threadIdx.x - 64;
        uint8_t* stg = smem + C::kStgOff + ew * 32 * stage_pitch<__nv_bfloat16>();
        __nv_bfloat16* Y = static_cast<__nv_bfloat16*>(ep.Y);
        const bool vec = ((static_cast<size_t>(N) * 2) % 16) == 0;
        const uint32_t tempty0 = dsmem_addr(tempty, 0);
        int i = 0;
        for (int t = pair; t < tiles; t += npairs, ++i) {
            const int ab = i & 1;
            const int use = i >> 1;
            const int m0 = (t / num_nt) * 2 * kQM + static_cast<int>(rank) * kQM;
            const int n0 = (t % num_nt) * kQN;
            // the tile's column tables (the last tile's reads are done)
            named_bar_sync(1, 32 * kQEpi);
            for (int e = et; e < kQN * RP; e += 32 * kQEpi) {
                const int col = e / RP, j = e % RP;
                const int n = n0 + col;
                sB[e] = (n < N && j < ep.r) ? __ldg(ep.B + static_cast<size_t>(j) * N + n) : 0.f;
            }
            for (int col = et; col < kQN; col += 32 * kQEpi) {
                const int n = n0 + col;
                sSw[col] = n < N ? __ldg(ep.sw + n) : 0.f;
                sBias[col] = (n < N && ep.bias) ? __ldg(ep.bias + n) : 0.f;
            }
            named_bar_sync(1, 32 * kQEpi);
            const int row0 = m0 + q * 32;
            const int row = row0 + lane;
            const bool row_ok = row < M;
            const float sxm = row_ok ? __ldg(ep.sx + row) : 0.f;
            float xa[RP];
#pragma unroll
            for (int j = 0; j < RP; ++j)
                xa[j] = (row_ok && j < ep.r) ? __ldg(ep.xA + static_cast<size_t>(row) * ep.r + j) * ep.c : 0.f;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[ab], use & 1, status));
            if (!ok) break;
            tc_fence_after();
            const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + ab * C::kAccCols;
#pragma unroll 1
            for (int col = 0; col < kQN; col += kEpiCols) {
                uint32_t v[kEpiCols];
                tmem_ld16(tbase + col, v);
                tmem_ld_wait();
                float y[kEpiCols];
#pragma unroll
                for (int e = 0; e < kEpiCols; ++e) {
                    const int c = col + e;
                    const float a = static_cast<float>(static_cast<int32_t>(v[e]));
                    float acc = fmaf(a * sxm, sSw[c], sBias[c]);
                    const float4* b4 = reinterpret_cast<const float4*>(sB + c * RP);
#pragma unroll
                    for (int j4 = 0; j4 < RP / 4; ++j4) {
                        const float4 b = b4[j4];
                        acc = fmaf(xa[4 * j4 + 0], b.x, acc);
                        acc = fmaf(xa[4 * j4 + 1], b.y, acc);
                        acc = fmaf(xa[4 * j4 + 2], b.z, acc);
                        acc = fmaf(xa[4 * j4 + 3], b.w, acc);
                    }
                    y[e] = acc;
                }
                if (ep.relu) {
#pragma unroll
                    for (int e = 0; e < kEpiCols; ++e) y[e] = y[e] > 0.f ? y[e] : 0.f;
                }
                if (ep.acc && row_ok) {
                    for (int e = 0; e < kEpiCols; ++e)
                        if (n0 + col + e < N)
                            ep.acc[static_cast<size_t>(row) * N + n0 + col + e] = static_cast<int32_t>(v[e]);
                }
                store_block<__nv_bfloat16>(stg, y, lane, Y, static_cast<size_t>(N), row0, M, n0 + col, N, vec);
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

template <int RP, bool W4>
cudaError_t launch_fwd_pair_t(const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                              const FwdEpilogue& ep, int* status, cudaStream_t s) {
    using C = PairFwdCfg<RP, W4>;
    auto kern = k2_gemm_i8_pair_kernel<RP, W4>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), C::kTotal);
    if (e != cudaSuccess) return e;
    CUtensorMap ta, tb;
    const bool bok = W4 ? make_tmap_2d(&tb, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, K / 2,
                                       kQN / 2, kQK / 2, CU_TENSOR_MAP_SWIZZLE_NONE)
                        : make_tmap_2d(&tb, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, K, kQN / 2, kQK,
                                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (!bok || !make_tmap_2d(&ta, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K, K, kQM, kQK,
                              CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int tiles = ((M + 2 * kQM - 1) / (2 * kQM)) * ((N + kQN - 1) / kQN);
    const int pairs = tiles < sm_count() / 2 ? tiles : sm_count() / 2;
    return launch_kx(kern, dim3(2 * pairs), dim3(q_threads<W4>()), C::kTotal, s, 2, ta, tb, M, N, K, ep,
                     status);
}

}  // namespace

bool gemm_fwd_pair_applies(Act act, int M, int N, int K, int r) {
    if (act != kBF16 || K % 16 != 0 || r > 16) return false;
    const int tiles = ((M + 2 * kQM - 1) / (2 * kQM)) * ((N + kQN - 1) / kQN);
    return tiles >= sm_count() / 2;
}

cudaError_t launch_gemm_i8_fwd_pair(const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                                    const FwdEpilogue& ep, int* status, cudaStream_t s, bool w4) {
    if (ep.r <= 4)
        return w4 ? launch_fwd_pair_t<4, true>(Xq, Wq, M, N, K, ep, status, s)
                  : launch_fwd_pair_t<4, false>(Xq, Wq, M, N, K, ep, status, s);
    if (ep.r <= 8)
        return w4 ? launch_fwd_pair_t<8, true>(Xq, Wq, M, N, K, ep, status, s)
                  : launch_fwd_pair_t<8, false>(Xq, Wq, M, N, K, ep, status, s);
    return w4 ? launch_fwd_pair_t<16, true>(Xq, Wq, M, N, K, ep, status, s)
              : launch_fwd_pair_t<16, false>(Xq, Wq, M, N, K, ep, status, s);
}

}  // namespace qlora
