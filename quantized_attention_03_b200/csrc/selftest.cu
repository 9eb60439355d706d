// Self-test of the bounded-wait path used by every mbarrier wait in the kernels: one
// thread waits on a barrier that nothing ever arrives on. The wait gives up after the
// requested time, records SAGE_ERR_TIMEOUT in the device status word and the kernel
// returns normally, leaving the context usable.
#include <cuda_runtime.h>

#include "sage_common.cuh"
#include "sm100_ptx.cuh"

namespace sage {
namespace {

__global__ void wait_selftest_kernel(int *status, uint64_t timeout_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        mbar_wait(&bar, 0, &abort, status, status_bit(SAGE_ERR_TIMEOUT), timeout_ns);
    __syncthreads();
}

}  // namespace

cudaError_t launch_wait_selftest(int *status, uint64_t timeout_ns, cudaStream_t st)
{
    wait_selftest_kernel<<<1, 32, 0, st>>>(status, timeout_ns);
    return cudaGetLastError();
}

}  // namespace sage
