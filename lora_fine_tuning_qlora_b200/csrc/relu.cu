// relu.cu -- the plain elementwise ReLU that sits between the Dense layers of
// the MNIST MLP ("Introduce QLoRA-like technique", benchmark.py: Dense +
// ReLU blocks).  Not part of the layer itself; kept as two in-place kernels.
#include "internal.h"
#include "ptx.cuh"

namespace qlora {

namespace {

template <typename T>
__global__ void relu_kernel(T* __restrict__ y, size_t n) {
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const float v = ActIO<T>::to_f(y[i]);
        if (!(v > 0.f)) y[i] = ActIO<T>::from_f(0.f);
    }
}

template <typename T>
__global__ void relu_backward_kernel(T* __restrict__ g, const T* __restrict__ h, size_t n) {
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        if (!(ActIO<T>::to_f(h[i]) > 0.f)) g[i] = ActIO<T>::from_f(0.f);
    }
}

int grid_for(size_t n) {
    size_t b = (n + 255) / 256;
    return static_cast<int>(b < 4 * 148 ? (b ? b : 1) : 4 * 148);
}

}  // namespace

cudaError_t launch_relu(Act act, void* y, size_t n, cudaStream_t s) {
    if (act == kBF16)
        relu_kernel<__nv_bfloat16><<<grid_for(n), 256, 0, s>>>(static_cast<__nv_bfloat16*>(y), n);
    else
        relu_kernel<float><<<grid_for(n), 256, 0, s>>>(static_cast<float*>(y), n);
    return cudaGetLastError();
}

cudaError_t launch_relu_backward(Act act, void* g, const void* h, size_t n, cudaStream_t s) {
    if (act == kBF16)
        relu_backward_kernel<__nv_bfloat16><<<grid_for(n), 256, 0, s>>>(
            static_cast<__nv_bfloat16*>(g), static_cast<const __nv_bfloat16*>(h), n);
    else
        relu_backward_kernel<float><<<grid_for(n), 256, 0, s>>>(static_cast<float*>(g),
                                                                static_cast<const float*>(h), n);
    return cudaGetLastError();
}

}  // namespace qlora
