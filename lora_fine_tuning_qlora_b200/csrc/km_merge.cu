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

// ---------------------------------------------------------------- tiled merge
// Ranks up to 8.  A CTA takes kNB = 8 output channels; each thread owns 16
// consecutive k (one 16-byte chunk of int8 codes, or 8 bytes of packed int4)
// per 4096-wide step of k and holds those rows of A in registers (eight at a
// time), so A is read once per CTA and sweep, and reused for all eight
// channels.  Sweep 1 forms w' and its per-channel abs-max, sweep 2 reads the
// codes again (mostly from L2), recomputes w' with the same operations and
// writes the new codes.  The arithmetic per element is the one of
// merged_value, in the same order, so the result is bit-identical to it.
constexpr int kNB = 8;
constexpr int kKStep = kThreads * 16;

// codes 8h .. 8h + 7 of a 16-code chunk (k order) -> exact floats, by
// placing each code (offset by 128) in the low mantissa byte of 2^23 and
// subtracting 2^23 + 128
__device__ __forceinline__ void codes_to_f8(const uint4 raw, int h, float (&f)[8]) {
    const uint32_t w0 = (h ? raw.z : raw.x) ^ 0x80808080u, w1 = (h ? raw.w : raw.y) ^ 0x80808080u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[i] = __fsub_rn(__uint_as_float(__byte_perm(w0, 0x4B000000u, 0x7540 + i)), 8388736.0f);
        f[4 + i] = __fsub_rn(__uint_as_float(__byte_perm(w1, 0x4B000000u, 0x7540 + i)), 8388736.0f);
    }
}

template <bool W4, int RP>
__global__ void __launch_bounds__(kThreads, RP <= 4 ? 2 : 1) km_merge_tiled_kernel(const uint8_t* __restrict__ Wq,
                                                                  const float* __restrict__ sw,
                                                                  const float* __restrict__ A,
                                                                  const float* __restrict__ B, int K,
                                                                  int N, int r, float c,
                                                                  uint8_t* __restrict__ Wq_out,
                                                                  float* __restrict__ sw_out) {
    constexpr float kLevels = W4 ? 7.0f : 127.0f;
    __shared__ float sB[RP][kNB];
    __shared__ float sS[kNB];
    __shared__ float red[kThreads / 32][kNB];
    __shared__ float s_amax[kNB];
    __shared__ float s_inv[kNB];  // kLevels / amax (0 for a zero channel)
    pdl_trigger();
    pdl_wait();
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int n0 = blockIdx.x * kNB;
    if (t < RP * kNB) {
        const int j = t / kNB, nb = t % kNB;
        sB[j][nb] = (j < r && n0 + nb < N) ? B[static_cast<size_t>(j) * N + n0 + nb] : 0.f;
    }
    if (t < kNB) sS[t] = n0 + t < N ? sw[n0 + t] : 0.f;
    __syncthreads();
    const size_t row_bytes = W4 ? static_cast<size_t>(K) / 2 : static_cast<size_t>(K);

    auto load_chunk = [&](int n, int k0) -> uint4 {
        const uint8_t* p = Wq + static_cast<size_t>(n) * row_bytes;
        if constexpr (W4) {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(p + k0 / 2));
            uint4 lo, hi;
            unpack_int4x32(make_uint4(v.x, v.y, 0u, 0u), lo, hi);
            return lo;  // codes k0 .. k0 + 15
        } else {
            return __ldg(reinterpret_cast<const uint4*>(p + k0));
        }
    };
    // A rows k0 .. k0 + 7
    auto load_a = [&](int k0, float (&a)[8][RP]) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
#pragma unroll
            for (int j = 0; j < RP; ++j)
                a[e][j] = j < r ? __ldg(A + static_cast<size_t>(k0 + e) * r + j) : 0.f;
    };
    // w'(k) for 8 k of channel nb (codes q), in the merge's fixed order
    auto merged8 = [&](const float* q, int nb, const float (&a)[8][RP], float (&wp)[8]) {
        const float s = sS[nb];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float w = __fmul_rn(q[e], s);
            float d = __fmul_rn(a[e][0], sB[0][nb]);
#pragma unroll
            for (int j = 1; j < RP; ++j)
                if (j < r) d = __fadd_rn(d, __fmul_rn(a[e][j], sB[j][nb]));
            wp[e] = __fadd_rn(w, __fmul_rn(c, d));
        }
    };

    float amax[kNB];
#pragma unroll
    for (int nb = 0; nb < kNB; ++nb) amax[nb] = 0.f;
    for (int ks = 0; ks < K; ks += kKStep) {
        const int k0 = ks + t * 16;
        if (k0 >= K) break;
        uint4 raw[kNB];
#pragma unroll
        for (int nb = 0; nb < kNB; ++nb)
            raw[nb] = n0 + nb < N ? load_chunk(n0 + nb, k0) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float a[8][RP];
            load_a(k0 + 8 * h, a);
#pragma unroll
            for (int nb = 0; nb < kNB; ++nb) {
                float q[8], wp[8];
                codes_to_f8(raw[nb], h, q);
                merged8(q, nb, a, wp);
#pragma unroll
                for (int e = 0; e < 8; ++e) amax[nb] = fmaxf(amax[nb], fabsf(wp[e]));
            }
        }
    }
    {
        const float x = xreduce<kNB, true>(amax);
        if ((lane & (32 / kNB - 1)) == 0) red[warp][xreduce_index<kNB>(lane)] = x;
    }
    __syncthreads();
    if (t < kNB) {
        float m = red[0][t];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[w][t]);
        s_amax[t] = m;
        s_inv[t] = m > 0.f ? __fdiv_rn(kLevels, m) : 0.f;
        if (n0 + t < N) sw_out[n0 + t] = __fdiv_rn(m, kLevels);
    }
    __syncthreads();

    for (int ks = 0; ks < K; ks += kKStep) {
        const int k0 = ks + t * 16;
        if (k0 >= K) break;
        uint4 raw[kNB];
#pragma unroll
        for (int nb = 0; nb < kNB; ++nb)
            raw[nb] = n0 + nb < N ? load_chunk(n0 + nb, k0) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float a[8][RP];
            load_a(k0 + 8 * h, a);
#pragma unroll
            for (int nb = 0; nb < kNB; ++nb) {
                const int n = n0 + nb;
                if (n >= N) break;
                float q[8], wp[8];
                codes_to_f8(raw[nb], h, q);
                merged8(q, nb, a, wp);
                const float inv = s_inv[nb];
                uint8_t* orow = Wq_out + static_cast<size_t>(n) * row_bytes;
                if constexpr (W4) {
                    uint32_t v = 0u;
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        v |= (static_cast<uint32_t>(quant_code_l<7>(wp[e], inv)) & 0xFu) << (4 * e);
                    *reinterpret_cast<uint32_t*>(orow + (k0 + 8 * h) / 2) = v;
                } else {
                    uint32_t v[2] = {0u, 0u};
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        v[e / 4] |= (static_cast<uint32_t>(quant_code(wp[e], inv)) & 0xFFu) << (8 * (e % 4));
                    *reinterpret_cast<uint2*>(orow + k0 + 8 * h) = make_uint2(v[0], v[1]);
                }
            }
        }
    }
}

template <bool W4>
cudaError_t launch_merge_t(const uint8_t* Wq, const float* sw, const float* A, const float* B,
                           int K, int N, int r, float c, uint8_t* Wq_out, float* sw_out,
                           cudaStream_t s) {
    const dim3 grid((N + kNB - 1) / kNB);
    if (r <= 4)
        return launch_k(km_merge_tiled_kernel<W4, 4>, grid, dim3(kThreads), 0, s, 1, Wq, sw, A, B, K,
                        N, r, c, Wq_out, sw_out);
    if (r <= 8)
        return launch_k(km_merge_tiled_kernel<W4, 8>, grid, dim3(kThreads), 0, s, 1, Wq, sw, A, B, K,
                        N, r, c, Wq_out, sw_out);
    km_merge_kernel<W4><<<N, kThreads, 0, s>>>(Wq, sw, A, B, K, N, r, c, Wq_out, sw_out);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge(const int8_t* Wq, const float* sw, const float* A, const float* B, int K,
                         int N, int r, float c, int8_t* Wq_out, float* sw_out, cudaStream_t s) {
    return launch_merge_t<false>(reinterpret_cast<const uint8_t*>(Wq), sw, A, B, K, N, r, c,
                                 reinterpret_cast<uint8_t*>(Wq_out), sw_out, s);
}

cudaError_t launch_merge_int4(const uint8_t* Wp, const float* sw, const float* A, const float* B,
                              int K, int N, int r, float c, uint8_t* Wp_out, float* sw_out,
                              cudaStream_t s) {
    return launch_merge_t<true>(Wp, sw, A, B, K, N, r, c, Wp_out, sw_out, s);
}

}  // namespace qlora
