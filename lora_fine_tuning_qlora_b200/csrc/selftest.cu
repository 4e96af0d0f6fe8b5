// selftest.cu -- exercises the bounded-wait failure path without faulting
// the GPU: one thread waits on an mbarrier that nothing arrives on, gives up
// after `limit_ns`, records the timeout in the device status word and exits
// normally.  The context stays usable; the host reads the status back.
#include "internal.h"
#include "ptx.cuh"

namespace qlora {

namespace {

__global__ void selftest_wait_kernel(int* status, unsigned long long limit_ns, int* waited) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // phase 0 never completes: nobody arrives
        const bool ok = mbar_wait(&bar, 0, status, limit_ns);
        if (waited) *waited = ok ? 0 : 1;
    }
}

}  // namespace

cudaError_t launch_selftest_wait(int* status, unsigned long long limit_ns, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(status, limit_ns, nullptr);
    return cudaGetLastError();
}

}  // namespace qlora
