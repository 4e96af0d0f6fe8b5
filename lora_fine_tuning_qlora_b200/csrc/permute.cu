// permute.cu -- axis permutation of a row-major tensor (up to 8 axes), the
// layout step of the EinsumDense equations that are not a Dense layer on a
// plain reshape ("Introduce float8 training": the EinsumDense speed test
// "abcde,aebf->adbcf"; "Introduce QLoRA-like technique": EinsumDense rows of
// the Results table).  An equation is brought to [batch, kept, contracted]
// operands before the layer and its output back to the equation's order
// after it.
//
// dst axis d is src axis perm[d]: dst[i_0, .., i_{n-1}] = src[j] with
// j_{perm[d]} = i_d.  One thread per destination element (consecutive
// threads write consecutive elements); the source offset is rebuilt from the
// destination index by a division per axis.  Elements of 1, 2, 4 or 8 bytes.
#include "internal.h"
#include "ptx.cuh"

namespace qlora {

namespace {

struct PermArgs {
    int nd;
    long long dst_dim[kMaxPermAxes];     // destination extents
    long long src_stride[kMaxPermAxes];  // source stride (elements) of the axis at each destination position
    long long n;
};

template <typename T>
__global__ void __launch_bounds__(256) permute_kernel(const T* __restrict__ src, T* __restrict__ dst, PermArgs a) {
    pdl_trigger();
    pdl_wait();
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < a.n; i += stride) {
        long long rem = i, off = 0;
        for (int d = a.nd - 1; d >= 0; --d) {
            const long long q = rem / a.dst_dim[d];
            off += (rem - q * a.dst_dim[d]) * a.src_stride[d];
            rem = q;
        }
        dst[i] = __ldg(src + off);
    }
}

}  // namespace

cudaError_t launch_permute(const void* src, void* dst, int nd, const long long* shape, const int* perm,
                           int elem_bytes, cudaStream_t s) {
    PermArgs a{};
    a.nd = nd;
    long long sstride[kMaxPermAxes];
    long long acc = 1;
    for (int d = nd - 1; d >= 0; --d) {
        sstride[d] = acc;
        acc *= shape[d];
    }
    a.n = acc;
    for (int d = 0; d < nd; ++d) {
        a.dst_dim[d] = shape[perm[d]];
        a.src_stride[d] = sstride[perm[d]];
    }
    if (a.n == 0) return cudaSuccess;
    const long long blocks = (a.n + 255) / 256;
    const int grid = static_cast<int>(blocks < 8LL * sm_count() ? blocks : 8LL * sm_count());
    switch (elem_bytes) {
        case 1: return launch_k(permute_kernel<uint8_t>, dim3(grid), dim3(256), 0, s, 1,
                                static_cast<const uint8_t*>(src), static_cast<uint8_t*>(dst), a);
        case 2: return launch_k(permute_kernel<uint16_t>, dim3(grid), dim3(256), 0, s, 1,
                                static_cast<const uint16_t*>(src), static_cast<uint16_t*>(dst), a);
        case 4: return launch_k(permute_kernel<uint32_t>, dim3(grid), dim3(256), 0, s, 1,
                                static_cast<const uint32_t*>(src), static_cast<uint32_t*>(dst), a);
        case 8: return launch_k(permute_kernel<unsigned long long>, dim3(grid), dim3(256), 0, s, 1,
                                static_cast<const unsigned long long*>(src), static_cast<unsigned long long*>(dst), a);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qlora
