// scratch.cu -- stream-ordered scratch for the forms that need a workspace
// (masked-parallel unknowns, the per-chunk images of the split chunk-parallel
// forward).  The memory comes from a pool the library owns, one per device,
// whose release threshold is unbounded: freed blocks stay mapped and are
// reused by the next call on any stream, instead of being handed back to the
// driver at every synchronisation and mapped again on the next call.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "kernels.h"

namespace falcon {

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_pool_mutex;
cudaMemPool_t g_pools[kMaxDevices];
bool g_pool_made[kMaxDevices];

cudaError_t device_pool(cudaMemPool_t *pool) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_pool_mutex);
    if (!g_pool_made[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        e = cudaMemPoolCreate(&g_pools[dev], &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = UINT64_MAX;
        e = cudaMemPoolSetAttribute(g_pools[dev], cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) return e;
        g_pool_made[dev] = true;
    }
    *pool = g_pools[dev];
    return cudaSuccess;
}

}  // namespace

cudaError_t scratch_alloc(void **ptr, size_t bytes, cudaStream_t s) {
    cudaMemPool_t pool;
    const cudaError_t e = device_pool(&pool);
    if (e != cudaSuccess) return e;
    return cudaMallocFromPoolAsync(ptr, bytes, pool, s);
}

cudaError_t scratch_free(void *ptr, cudaStream_t s) { return cudaFreeAsync(ptr, s); }

cudaError_t scratch_trim() {
    cudaMemPool_t pool;
    const cudaError_t e = device_pool(&pool);
    if (e != cudaSuccess) return e;
    return cudaMemPoolTrimTo(pool, 0);
}

}  // namespace falcon
