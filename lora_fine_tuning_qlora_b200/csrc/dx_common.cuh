// dx_common.cuh -- pieces shared by the two dX GEMM kernels (k3_dx.cu and
// k3_dx_pair.cu): the MN-major 128-byte-swizzled layout of the de-quantized
// kernel tile, the conversion of int8 codes to bf16(q * scale), and the G
// rows of the rank-r term.
#pragma once

#include "internal.h"
#include "ptx.cuh"

#include <cuda_fp16.h>

namespace qlora {

// byte offset of the 16-byte chunk holding bf16 elements (mn .. mn+7, kr) in
// an MN-major, 128B-swizzled operand tile with 8-row K groups 1024 B apart and
// 64-element MN blocks `lbo` bytes apart.
__device__ __forceinline__ uint32_t mn_sw128_offset(int mn, int kr, uint32_t lbo) {
    const int mb = mn >> 6;
    const int chunk = (mn & 63) >> 3;
    const int kg = kr >> 3;
    const int row = kr & 7;
    return mb * lbo + kg * 1024 + row * 128 + ((chunk ^ row) << 4);
}

// Chunk c of a de-quantize stage -> (contraction row nr, 16-byte chunk kc of
// that row), CPR chunks per row.  With 8 chunks per row (two 64-element MN
// blocks) the plain row-major order puts chunks kc and kc + 4 of one row,
// which land on the same shared-memory banks one MN block apart, in the same
// 8-lane phase of a 16-byte store; instead every 8 consecutive chunks cover
// two rows of opposite parity and four chunks of one MN block, so the
// swizzled positions ((kc % 4) * 2 ^ row) of a phase are all distinct.  The
// rows a warp covers are the same set as in row-major order.
template <int CPR>
__device__ __forceinline__ void chunk_rc(int c, int& nr, int& kc) {
    if constexpr (CPR == 8) {
        const int rest = c >> 3;
        nr = 2 * (rest >> 1) + ((c >> 2) & 1);
        kc = (c & 3) + 4 * (rest & 1);
    } else {
        nr = c / CPR;
        kc = c % CPR;
    }
}

// G[m,j] = sum over the column-block slices of G (fixed order).
__device__ __forceinline__ float g_row(const DxEpilogue& ep, int M, int m, int j) {
    return sum_slices(ep.Gp + static_cast<size_t>(m) * ep.r + j, static_cast<size_t>(M) * ep.r,
                      ep.ncb);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ unsigned long long f2(float a, float b) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}

// 16 int8 codes (one 16-byte chunk, element i in byte i) -> 8 words of packed
// bf16 pairs holding bf16(fl32(q * scale)).  Each code becomes the exact
// float 2^23 + (q + 128) by a byte permute into 0x4B000000, an exact add of
// -(2^23 + 128) recovers q, then one fp32 multiply by the scale (pairs of
// lanes in f32x2 instructions) and a round-to-nearest-even to bf16 in integer
// ALU operations: the same value as converting q to float, multiplying and
// converting to bf16, without the conversion pipe.
__device__ __forceinline__ void dequant16(const uint4 raw, float scale, uint32_t (&o)[8]) {
    const uint32_t w[4] = {raw.x ^ 0x80808080u, raw.y ^ 0x80808080u, raw.z ^ 0x80808080u,
                           raw.w ^ 0x80808080u};
    const unsigned long long bias2 = f2(-8388736.0f, -8388736.0f);
    const unsigned long long sc2 = f2(scale, scale);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        unsigned long long lo = f2(__uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7540)),
                                   __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7541)));
        unsigned long long hi = f2(__uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7542)),
                                   __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7543)));
        asm("add.rn.f32x2 %0, %0, %1;" : "+l"(lo) : "l"(bias2));
        asm("add.rn.f32x2 %0, %0, %1;" : "+l"(hi) : "l"(bias2));
        asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(lo) : "l"(sc2));
        asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(hi) : "l"(sc2));
        float a, b, c, d;
        asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(lo));
        asm("mov.b64 {%0, %1}, %2;" : "=f"(c), "=f"(d) : "l"(hi));
        o[2 * i] = pack_bf16x2(a, b);
        o[2 * i + 1] = pack_bf16x2(c, d);
    }
}

// Element (k, j) of the rank-r epilogue's factor (A for dX; B^T for a forward
// run on the dX kernels).
__device__ __forceinline__ float a_at(const DxEpilogue& ep, int k, int j) {
    return __ldg(ep.A + static_cast<size_t>(k) * (ep.a_ks ? ep.a_ks : ep.r) +
                 static_cast<size_t>(j) * ep.a_js);
}

// 16 uint8 affine codes -> 8 words of packed bf16 pairs holding
// bf16(fl32(bias + fl32(code * scale))) (the rebuilt outlier-compensated
// kernel; the two roundings stay separate, as the reading fixes).
__device__ __forceinline__ void dequant16_affine(const uint4 raw, float scale, float bias,
                                                 uint32_t (&o)[8]) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float v[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const float code = __fsub_rn(__uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7540 + b)),
                                         8388608.0f);
            v[b] = __fadd_rn(bias, __fmul_rn(code, scale));
        }
        o[2 * i] = pack_bf16x2(v[0], v[1]);
        o[2 * i + 1] = pack_bf16x2(v[2], v[3]);
    }
}

// Writes the outliers of contraction row `row` (global), columns
// [c0, c0 + width) of the layout (c0 % 128 + width <= 128), into a stage's
// MN-major 128B-swizzled bf16 tile at contraction row `nr` (column c0 -> 0).
__device__ __forceinline__ void patch_outliers(const OutlierArgs& ol, int row, int c0, int width,
                                               uint8_t* tile, int nr, uint32_t lbo) {
    const int blk = c0 >> 7, off = c0 & 127;
    const size_t b = static_cast<size_t>(row) * ol.nb + blk;
    const int e0 = __ldg(ol.start + b), e1 = __ldg(ol.start + b + 1);
    for (int e = e0; e < e1; ++e) {
        const uint32_t v = __ldg(ol.ent + e);
        const int col = static_cast<int>(v >> 16) - off;
        if (col < 0 || col >= width) continue;
        const float f = __half2float(__ushort_as_half(static_cast<unsigned short>(v & 0xFFFFu)));
        *reinterpret_cast<__nv_bfloat16*>(tile + mn_sw128_offset(col & ~7, nr, lbo) + (col & 7) * 2) =
            __float2bfloat16_rn(f);
    }
}

}  // namespace qlora
