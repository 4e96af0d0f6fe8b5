// tile_epilogue.cuh -- pieces shared by the two tensor-core GEMM kernels:
// persistent tile scheduling, named barriers among the epilogue warps, and
// the staged, coalesced store of a 32-row x 16-column block of outputs that
// one epilogue warp reads from TMEM (one row per lane).
#pragma once

#include "ptx.cuh"

namespace qlora {

// Columns per TMEM load in the epilogue (tcgen05.ld.32x32b.x16).
constexpr int kEpiCols = 16;

// Bytes per staged row: 16 outputs plus 16 bytes of padding, which keeps
// both the per-lane row writes and the cooperative reads conflict-light.
template <typename OutT>
__host__ __device__ constexpr int stage_pitch() {
    return kEpiCols * static_cast<int>(sizeof(OutT)) + 16;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint32_t pack2(float a, float b, __nv_bfloat16*) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Writes the 16 values of this lane's row into the warp's staging buffer,
// then the warp stores the 32 x 16 block to global memory with 16-byte
// stores (rows row0 .. row0+31, columns n .. n+15 of a row-major [M, ldo]
// matrix).  Rows >= M or < row_min and columns >= N are skipped; when `vec` is false
// (row pitch not a multiple of 16 bytes) the copy-out is element by element.
template <typename OutT>
__device__ __forceinline__ void store_block(uint8_t* stg, const float (&v)[kEpiCols], int lane,
                                            OutT* __restrict__ out, size_t ldo, int row0, int M,
                                            int n, int N, bool vec, int row_min = 0) {
    constexpr int P = stage_pitch<OutT>();
    uint8_t* my = stg + lane * P;
    if constexpr (sizeof(OutT) == 2) {
        uint4 a, b;
        a.x = pack2(v[0], v[1], (__nv_bfloat16*)nullptr);
        a.y = pack2(v[2], v[3], (__nv_bfloat16*)nullptr);
        a.z = pack2(v[4], v[5], (__nv_bfloat16*)nullptr);
        a.w = pack2(v[6], v[7], (__nv_bfloat16*)nullptr);
        b.x = pack2(v[8], v[9], (__nv_bfloat16*)nullptr);
        b.y = pack2(v[10], v[11], (__nv_bfloat16*)nullptr);
        b.z = pack2(v[12], v[13], (__nv_bfloat16*)nullptr);
        b.w = pack2(v[14], v[15], (__nv_bfloat16*)nullptr);
        reinterpret_cast<uint4*>(my)[0] = a;
        reinterpret_cast<uint4*>(my)[1] = b;
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            reinterpret_cast<float4*>(my)[i] =
                make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
    __syncwarp();
    constexpr int kChunks = kEpiCols * static_cast<int>(sizeof(OutT)) / 16;  // per row
    constexpr int kRowsPerIt = 32 / kChunks;
    constexpr int kElems = 16 / static_cast<int>(sizeof(OutT));              // per chunk
#pragma unroll
    for (int it = 0; it < 32 / kRowsPerIt; ++it) {
        const int rr = it * kRowsPerIt + lane / kChunks;
        const int ch = lane % kChunks;
        const int gr = row0 + rr;
        const int gn = n + ch * kElems;
        if (gr < M && gr >= row_min && gn < N) {
            const uint4 val = *reinterpret_cast<const uint4*>(stg + rr * P + ch * 16);
            OutT* dst = out + static_cast<size_t>(gr) * ldo + gn;
            if (vec && gn + kElems <= N) {
                *reinterpret_cast<uint4*>(dst) = val;
            } else {
                const OutT* e = reinterpret_cast<const OutT*>(&val);
                for (int i = 0; i < kElems; ++i)
                    if (gn + i < N) dst[i] = e[i];
            }
        }
    }
    __syncwarp();
}

// Number of SMs of the current device (cached per device).
int sm_count();

}  // namespace qlora
