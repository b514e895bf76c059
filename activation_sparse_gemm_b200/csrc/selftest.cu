// Self-test of the bounded device-side waits: one thread waits on an mbarrier
// that nothing arrives on.  The wait gives up after limit_ns, records the
// timeout in the device error word and the kernel returns normally, so the
// CUDA context stays usable.
#include "internal.h"
#include "ptx.cuh"

namespace rtlynx {

__global__ void rtlynx_wait_selftest_kernel(int* err, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, err, limit_ns);  // never completes: times out
    __syncthreads();
}

int launch_wait_selftest(int* err, uint64_t limit_ns, cudaStream_t stream) {
    rtlynx_wait_selftest_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
    return cudaGetLastError();
}

}  // namespace rtlynx
