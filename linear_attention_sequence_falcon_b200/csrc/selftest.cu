// selftest.cu -- on-device check of the bounded waits used by the
// tensor-core kernels: a block waits on an mbarrier phase that nothing will
// ever complete and must give up after its time limit, report that, and
// leave normally (no fault, no hang; the context stays usable).
#include <cuda_runtime.h>

#include "../../include/falcon.h"
#include "kernels.h"
#include "tc_sm100.cuh"

namespace {

__device__ int g_selftest_result;

__global__ void bounded_wait_kernel(unsigned long long timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        falcon::tc::mbar_init(&bar, 1);  // expects one arrival that never comes
        falcon::tc::fence_mbar_init();
    }
    __syncthreads();
    const bool done = falcon::tc::mbar_wait_timeout(&bar, 0, timeout_ns);
    const int gave_up = __syncthreads_or(!done);
    if (threadIdx.x == 0) g_selftest_result = gave_up ? 1 : 0;
}

}  // namespace

extern "C" int falcon_selftest_bounded_wait(unsigned int timeout_us, int *gave_up) {
    if (!gave_up) return FALCON_ERR_NULL;
    const int minus_one = -1;
    if (cudaMemcpyToSymbol(g_selftest_result, &minus_one, sizeof(int)) != cudaSuccess) return FALCON_ERR_LAUNCH;
    bounded_wait_kernel<<<1, 64>>>(1000ull * timeout_us);
    if (cudaGetLastError() != cudaSuccess) return FALCON_ERR_LAUNCH;
    if (cudaMemcpyFromSymbol(gave_up, g_selftest_result, sizeof(int)) != cudaSuccess) return FALCON_ERR_LAUNCH;
    return FALCON_OK;
}
