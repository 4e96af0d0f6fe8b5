// relu.cu -- the plain elementwise ReLU that sits between the Dense layers of
// the MNIST MLP ("Introduce QLoRA-like technique", benchmark.py: Dense +
// ReLU blocks).  Not part of the layer itself; kept as two in-place kernels,
// 16-byte vectors when the buffers allow it.
#include "internal.h"
#include "ptx.cuh"

namespace qlora {

namespace {

template <typename T>
__device__ __forceinline__ bool positive(T v) {
    return ActIO<T>::to_f(v) > 0.f;
}

template <typename T>
__global__ void relu_kernel(T* __restrict__ y, size_t n, bool vec) {
    pdl_trigger();
    pdl_wait();
    constexpr int kV = 16 / sizeof(T);
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
    if (vec) {
        const size_t nv = n / kV;
        for (; i < nv; i += stride) {
            uint4 u = reinterpret_cast<uint4*>(y)[i];
            T* e = reinterpret_cast<T*>(&u);
#pragma unroll
            for (int k = 0; k < kV; ++k)
                if (!positive(e[k])) e[k] = ActIO<T>::from_f(0.f);
            reinterpret_cast<uint4*>(y)[i] = u;
        }
        i = nv * kV + blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
    }
    for (; i < n; i += stride)
        if (!positive(y[i])) y[i] = ActIO<T>::from_f(0.f);
}

template <typename T>
__global__ void relu_backward_kernel(T* __restrict__ g, const T* __restrict__ h, size_t n, bool vec) {
    pdl_trigger();
    pdl_wait();
    constexpr int kV = 16 / sizeof(T);
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
    if (vec) {
        const size_t nv = n / kV;
        for (; i < nv; i += stride) {
            uint4 u = reinterpret_cast<uint4*>(g)[i];
            const uint4 hv = reinterpret_cast<const uint4*>(h)[i];
            T* e = reinterpret_cast<T*>(&u);
            const T* he = reinterpret_cast<const T*>(&hv);
#pragma unroll
            for (int k = 0; k < kV; ++k)
                if (!positive(he[k])) e[k] = ActIO<T>::from_f(0.f);
            reinterpret_cast<uint4*>(g)[i] = u;
        }
        i = nv * kV + blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
    }
    for (; i < n; i += stride)
        if (!positive(h[i])) g[i] = ActIO<T>::from_f(0.f);
}

int grid_for(size_t work) {
    size_t b = (work + 255) / 256;
    const size_t cap = 8 * static_cast<size_t>(sm_count());
    return static_cast<int>(b < 1 ? 1 : (b > cap ? cap : b));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

cudaError_t launch_relu(Act act, void* y, size_t n, cudaStream_t s) {
    const bool vec = aligned16(y);
    if (act == kBF16)
        return launch_k(relu_kernel<__nv_bfloat16>, dim3(grid_for(n / 8 + 1)), dim3(256), 0, s, 1,
                        static_cast<__nv_bfloat16*>(y), n, vec);
    return launch_k(relu_kernel<float>, dim3(grid_for(n / 4 + 1)), dim3(256), 0, s, 1,
                    static_cast<float*>(y), n, vec);
}

cudaError_t launch_relu_backward(Act act, void* g, const void* h, size_t n, cudaStream_t s) {
    const bool vec = aligned16(g) && aligned16(h);
    if (act == kBF16)
        return launch_k(relu_backward_kernel<__nv_bfloat16>, dim3(grid_for(n / 8 + 1)), dim3(256), 0, s,
                        1, static_cast<__nv_bfloat16*>(g), static_cast<const __nv_bfloat16*>(h), n, vec);
    return launch_k(relu_backward_kernel<float>, dim3(grid_for(n / 4 + 1)), dim3(256), 0, s, 1,
                    static_cast<float*>(g), static_cast<const float*>(h), n, vec);
}

}  // namespace qlora
