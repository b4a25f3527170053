// scratch.cu -- the workspace of the forms that need one (masked-parallel
// unknowns, the per-chunk images of the split chunk-parallel forward, the
// Falcon-2A state images, the backward's per-token arrays).
//
// A call either runs in a workspace its caller hands in (the *_ws entry
// points: the library then allocates nothing) or, for the allocating entry
// points, draws the workspace stream-ordered from the device's current memory
// pool (cudaMallocAsync; the runtime's default pool unless the caller has set
// another) and frees it on the same stream at the end of the call's work.
// The library keeps no pool of its own: whatever the pool retains between
// calls follows the pool's release threshold, which belongs to the caller.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace falcon {

cudaError_t scratch_alloc(void **ptr, size_t bytes, cudaStream_t s) { return cudaMallocAsync(ptr, bytes, s); }

cudaError_t scratch_free(void *ptr, cudaStream_t s) { return cudaFreeAsync(ptr, s); }

cudaError_t scratch_trim() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    cudaMemPool_t pool;
    e = cudaDeviceGetMemPool(&pool, dev);
    if (e != cudaSuccess) return e;
    return cudaMemPoolTrimTo(pool, 0);
}

int ws_acquire(int given, void *given_ptr, size_t given_bytes, size_t need, cudaStream_t s, void **ptr,
               bool *owned) {
    *ptr = nullptr;
    *owned = false;
    if (given) {
        if (need == 0) return 0;
        if (!given_ptr || given_bytes < need || (reinterpret_cast<uintptr_t>(given_ptr) & 255u) != 0)
            return kErrWorkspace;
        *ptr = given_ptr;
        return 0;
    }
    if (need == 0) return 0;
    if (scratch_alloc(ptr, need, s) != cudaSuccess) {
        cudaGetLastError();
        *ptr = nullptr;
        return kErrAlloc;
    }
    *owned = true;
    return 0;
}

void ws_release(void *ptr, bool owned, cudaStream_t s) {
    if (owned && ptr) scratch_free(ptr, s);
}

}  // namespace falcon
