// Check of the failure path the kernels rely on: a bounded wait that is never
// satisfied gives up after its limit, records the timeout bit in the device
// error word and returns, and the context stays usable. No fault, trap or hang
// is involved: the two waits below are the same helpers the pipelines use,
// pointed at an mbarrier phase that no thread completes and at a counter that
// nothing increments.
#include "common.cuh"
#include "moge_internal.h"

namespace moge {

__global__ void wait_selftest_kernel(int32_t *out, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival expected; none comes
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        out[0] = mbar_wait(&bar, 0u, nullptr, limit_ns) ? 0 : 1;
        out[1] = wait_counter(out + 2, 1, nullptr, limit_ns) ? 0 : 1;  // out[2] stays 0
    }
}

cudaError_t launch_wait_selftest(int32_t *out, uint64_t limit_ns, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(out, 0, 3 * sizeof(int32_t), st);
    if (e != cudaSuccess) return e;
    wait_selftest_kernel<<<1, 32, 0, st>>>(out, limit_ns);
    return cudaGetLastError();
}

}  // namespace moge
