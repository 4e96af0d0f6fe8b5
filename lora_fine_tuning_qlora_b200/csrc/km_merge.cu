// km_merge.cu -- the lossy merge of the LoRA adapter into the int8 kernel
// ("Introduce QLoRA-like technique", Results footnote: merging LoRA weights
// into int8 kernels is lossy; "How to fine-tune the 4-bit model?" thread:
// de-quantize, add the LoRA, re-quantize; the float increment is
// einsum(A, B) * alpha / rank, "Merge weights and generate text!").
//
// One CTA per output channel n (a row of Wq [N,K], contiguous in K; or of
// the packed int4 codes [N, K/2], re-quantized to int4 with 7 levels):
//   w'(k) = fl(fl(q * s) + fl(c * d)),  d = A[k,0]B[0,n] + ... (ascending j)
// pass 1 takes the abs-max of w' over k, pass 2 recomputes w' with the same
// operations (bit-identical) and quantizes it.  Every operation is a single
// IEEE fp32 rounding (__fmul_rn / __fadd_rn / __fdiv_rn), so the result is
// bit-exact with that order.  HBM-bound: Wq is read from HBM once (pass 2
// hits L2), Wq_out is written once; A is shared by all CTAs through L2.
#include "internal.h"
#include "ptx.cuh"

namespace qlora {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float merged_value(int8_t q, float s, const float* __restrict__ arow,
                                              const float* __restrict__ bcol, int r, float c) {
    const float w = __fmul_rn(static_cast<float>(q), s);
    float d = __fmul_rn(__ldg(arow), bcol[0]);
    for (int j = 1; j < r; ++j) d = __fadd_rn(d, __fmul_rn(__ldg(arow + j), bcol[j]));
    return __fadd_rn(w, __fmul_rn(c, d));
}

// W4 = false: int8 codes in and out (127 levels); W4 = true: packed int4
// codes in and out (7 levels, two per byte, even k in the low nibble), so a
// chunk of 16 bytes holds 16 or 32 codes.
template <bool W4>
__global__ void __launch_bounds__(kThreads) km_merge_kernel(const uint8_t* __restrict__ Wq,
                                                            const float* __restrict__ sw,
                                                            const float* __restrict__ A,
                                                            const float* __restrict__ B, int K,
                                                            int N, int r, float c,
                                                            uint8_t* __restrict__ Wq_out,
                                                            float* __restrict__ sw_out) {
    constexpr int kCodes = W4 ? 32 : 16;      // codes per 16-byte chunk
    constexpr float kLevels = W4 ? 7.0f : 127.0f;
    __shared__ float bcol[64];
    __shared__ float red[kThreads / 32];
    const int n = blockIdx.x;
    const int t = threadIdx.x;
    if (t < r) bcol[t] = B[static_cast<size_t>(t) * N + n];
    __syncthreads();
    const float s = sw[n];
    const size_t row_bytes = W4 ? static_cast<size_t>(K) / 2 : static_cast<size_t>(K);
    const uint8_t* qrow = Wq + static_cast<size_t>(n) * row_bytes;
    // the chunk's codes as int8, in k order
    auto load_codes = [&](int k0, int8_t (&q)[kCodes]) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(qrow + (W4 ? k0 / 2 : k0)));
        if constexpr (W4) {
            uint4 lo, hi;
            unpack_int4x32(raw, lo, hi);
            *reinterpret_cast<uint4*>(q) = lo;
            *reinterpret_cast<uint4*>(q + 16) = hi;
        } else {
            *reinterpret_cast<uint4*>(q) = raw;
        }
    };

    float amax = 0.f;
    for (int k0 = t * kCodes; k0 < K; k0 += kThreads * kCodes) {
        alignas(16) int8_t q[kCodes];
        load_codes(k0, q);
#pragma unroll
        for (int e = 0; e < kCodes; ++e)
            amax = fmaxf(amax, fabsf(merged_value(q[e], s, A + static_cast<size_t>(k0 + e) * r, bcol, r, c)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((t & 31) == 0) red[t >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < kThreads / 32; ++i) amax = fmaxf(amax, red[i]);
    const float inv = amax > 0.f ? __fdiv_rn(kLevels, amax) : 0.f;
    if (t == 0) sw_out[n] = __fdiv_rn(amax, kLevels);

    uint8_t* orow = Wq_out + static_cast<size_t>(n) * row_bytes;
    for (int k0 = t * kCodes; k0 < K; k0 += kThreads * kCodes) {
        alignas(16) int8_t q[kCodes];
        load_codes(k0, q);
        uint32_t o[4] = {0, 0, 0, 0};
#pragma unroll
        for (int e = 0; e < kCodes; ++e) {
            const float w = merged_value(q[e], s, A + static_cast<size_t>(k0 + e) * r, bcol, r, c);
            if constexpr (W4)
                o[e / 8] |= (static_cast<uint32_t>(quant_code_l<7>(w, inv)) & 0xFu) << (4 * (e % 8));
            else
                o[e / 4] |= (static_cast<uint32_t>(quant_code(w, inv)) & 0xFFu) << (8 * (e % 4));
        }
        *reinterpret_cast<uint4*>(orow + (W4 ? k0 / 2 : k0)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace

cudaError_t launch_merge(const int8_t* Wq, const float* sw, const float* A, const float* B, int K,
                         int N, int r, float c, int8_t* Wq_out, float* sw_out, cudaStream_t s) {
    km_merge_kernel<false><<<N, kThreads, 0, s>>>(reinterpret_cast<const uint8_t*>(Wq), sw, A, B, K,
                                                  N, r, c, reinterpret_cast<uint8_t*>(Wq_out), sw_out);
    return cudaGetLastError();
}

cudaError_t launch_merge_int4(const uint8_t* Wp, const float* sw, const float* A, const float* B,
                              int K, int N, int r, float c, uint8_t* Wp_out, float* sw_out,
                              cudaStream_t s) {
    km_merge_kernel<true><<<N, kThreads, 0, s>>>(Wp, sw, A, B, K, N, r, c, Wp_out, sw_out);
    return cudaGetLastError();
}

}  // namespace qlora
