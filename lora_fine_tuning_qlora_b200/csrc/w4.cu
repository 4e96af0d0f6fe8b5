// w4.cu -- packed int4 frozen kernels: the one-off quantization of a float
// kernel into 4-bit codes, two per byte, and their expansion to int8 codes.
//
// keras-llm-light ("Simplified Int4Variable quantization") stores two int4
// values in one int8 byte to halve the kernel's memory; the "How to fine-tune
// the 4-bit model?" thread trains an fp32 LoRA over a frozen 4-bit kernel.
// Reading: the int8 quantizer with 7 in place of 127, per output channel n:
//   s[n] = amax / 7,  q[n,k] = clamp(rne(W[k,n] * (7 / amax)), -7, 7)
// in fp32 with one rounding per operation; byte j of channel n holds code 2j
// in its low nibble and code 2j+1 in its high nibble (two's complement).
// An int4 layer computes what the int8 layer computes with these codes: its
// dX GEMM de-quantizes the nibbles in shared memory (k3_dx.cu); its forward
// runs the int8 GEMM on the codes expanded by k_unpack_int4_kernel.
#include "internal.h"
#include "ptx.cuh"

namespace qlora {

namespace {

constexpr int kQwCols = 32;
constexpr int kQwK = 128;

// One CTA per 32 output channels: column abs-max, then 128 x 32 tiles
// transposed through shared memory so that each thread packs 16 consecutive
// codes of one channel into 8 bytes of its row.
__global__ void __launch_bounds__(256) k_quantize_weight_int4_kernel(const float* __restrict__ W,
                                                                     int K, int N,
                                                                     uint8_t* __restrict__ Wp,
                                                                     float* __restrict__ sw) {
    __shared__ float part[8][kQwCols];
    __shared__ float inv_s[kQwCols];
    __shared__ float tile[kQwK][kQwCols + 1];
    const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;
    const int n0 = blockIdx.x * kQwCols;
    const int n = n0 + tx;
    float amax = 0.f;
    if (n < N)
        for (int k = ty; k < K; k += 8) amax = fmaxf(amax, fabsf(__ldg(W + static_cast<size_t>(k) * N + n)));
    part[ty][tx] = amax;
    __syncthreads();
    if (ty == 0) {
        float a = part[0][tx];
#pragma unroll
        for (int i = 1; i < 8; ++i) a = fmaxf(a, part[i][tx]);
        inv_s[tx] = a > 0.f ? __fdiv_rn(7.0f, a) : 0.f;
        if (n < N) sw[n] = __fdiv_rn(a, 7.0f);
    }
    __syncthreads();
    const size_t row_bytes = static_cast<size_t>(K) / 2;
    for (int k0 = 0; k0 < K; k0 += kQwK) {
        for (int kk = ty; kk < kQwK; kk += 8) {
            const int k = k0 + kk;
            tile[kk][tx] = (n < N && k < K) ? __ldg(W + static_cast<size_t>(k) * N + n) : 0.f;
        }
        __syncthreads();
        // 256 threads cover 32 channels x 8 groups of 16 consecutive k
        const int c = threadIdx.x / 8;
        const int g = threadIdx.x % 8;
        const int nn = n0 + c;
        const int kb = k0 + g * 16;  // K is a multiple of 32: a group is all in or all out
        if (nn < N && kb < K) {
            const float inv = inv_s[c];
            uint32_t w[2] = {0u, 0u};
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const uint32_t code = static_cast<uint32_t>(quant_code_l<7>(tile[g * 16 + e][c], inv)) & 0xFu;
                w[e / 8] |= code << (4 * (e % 8));
            }
            *reinterpret_cast<uint2*>(Wp + static_cast<size_t>(nn) * row_bytes + kb / 2) = make_uint2(w[0], w[1]);
        }
        __syncthreads();
    }
}

// Wp [N, K/2] packed codes -> Wq [N, K] int8 codes; one 16-byte chunk (32
// codes) per thread and step.
__global__ void __launch_bounds__(256) k_unpack_int4_kernel(const uint8_t* __restrict__ Wp,
                                                            size_t chunks, int8_t* __restrict__ Wq) {
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < chunks;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        uint4 lo, hi;
        unpack_int4x32(__ldg(reinterpret_cast<const uint4*>(Wp) + i), lo, hi);
        reinterpret_cast<uint4*>(Wq)[2 * i] = lo;
        reinterpret_cast<uint4*>(Wq)[2 * i + 1] = hi;
    }
}

}  // namespace

cudaError_t launch_quantize_weight_int4(const float* W, int K, int N, uint8_t* Wp, float* sw,
                                        cudaStream_t s) {
    k_quantize_weight_int4_kernel<<<(N + kQwCols - 1) / kQwCols, 256, 0, s>>>(W, K, N, Wp, sw);
    return cudaGetLastError();
}

cudaError_t launch_unpack_int4(const uint8_t* Wp, int K, int N, int8_t* Wq, cudaStream_t s) {
    const size_t chunks = static_cast<size_t>(N) * K / 32;
    size_t blocks = (chunks + 255) / 256;
    const size_t cap = static_cast<size_t>(sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks == 0) return cudaSuccess;
    k_unpack_int4_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(Wp, chunks, Wq);
    return cudaGetLastError();
}

}  // namespace qlora
