// A device-side check of the kernels' failure path: the bounded pipeline wait.
//
// Every wait in the library's kernels gives up after a time limit instead of
// spinning forever, raises PA_DEV_WAIT_TIMEOUT in the status word and lets the
// kernel return, so a stalled pipeline surfaces as a status bit the host reads
// while the context stays usable.  This kernel makes such a wait run out on
// purpose: one thread waits on an mbarrier that nothing ever arrives at, with the
// same helper and limit the kernels use.  Nothing faults, traps or hangs.
#include <cuda_runtime.h>

#include <cstdint>

#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {
namespace {

__device__ unsigned long long g_selftest_waited_ns;

__global__ void bounded_wait_selftest_kernel(unsigned int* status)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival expected, none will come
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned long long t0 = globaltimer_ns();
        if (!mbar_wait_bounded(&bar, 0, &abort_flag)) atomicOr(status, PA_DEV_WAIT_TIMEOUT);
        g_selftest_waited_ns = globaltimer_ns() - t0;
    }
}

}  // namespace

cudaError_t launch_wait_selftest(unsigned int* status, unsigned long long* waited_ns, cudaStream_t stream)
{
    bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbolAsync(waited_ns, g_selftest_waited_ns, sizeof(unsigned long long), 0,
                                  cudaMemcpyDeviceToHost, stream);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(stream);
}

}  // namespace pa
