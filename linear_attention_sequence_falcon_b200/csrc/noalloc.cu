// noalloc.cu -- falcon_fwd_masked_noalloc: the masked-parallel forward with
// its scratch in a fixed, library-owned device array instead of memory
// obtained from the allocator.
//
// Why it exists: some callers of this library may not allocate device
// memory at all -- a host that owns every device allocation and hands a
// plug-in only its input and output buffers, or a server that runs under a
// fixed, pre-planned memory budget where an allocation at call time is not
// allowed.  falcon_fwd's masked form needs scratch (the solved unknowns, the
// steps and the cumulative log decay of every token), which it draws with
// cudaMallocAsync; this entry point draws the same scratch from the array
// below and makes no allocation of any kind.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library's device code holds its kNoAllocScratchBytes until the process
// exits.  With lazy module loading (the CUDA 12 default) the array is
// materialised when the module is first loaded on a device, which may be
// inside this entry point's first call there: a caller on a fixed budget
// should make that first call during set-up, before the budget is fixed.
// Host code may not use the array's name as a device address (on the host it
// names a stand-in object), so the device address is looked up once per
// device with cudaGetSymbolAddress, with that device current, on the first
// call that runs on it; that first call should therefore come before any
// stream capture.  A lookup that fails for lack of memory returns
// FALCON_ERR_ALLOC.  All calls on a device share the one array: calls that overlap on
// the GPU (different streams, or several host threads) race on it and must
// be serialised by the caller.  The kernel writes every scratch element
// before reading it, so nothing needs clearing between calls.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/falcon.h"
#include "common.cuh"
#include "kernels.h"

using namespace falcon;

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)FALCON_NOALLOC_SCRATCH_BYTES;
constexpr size_t kNoAllocScratchFloats = kNoAllocScratchBytes / sizeof(float);
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_scratch[kNoAllocScratchFloats];

std::mutex g_mu;
float *g_addr[kMaxDevices];  // device address of g_scratch, per device ordinal

int scratch_address(float **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return FALCON_ERR_LAUNCH;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return e == cudaErrorMemoryAllocation ? FALCON_ERR_ALLOC : FALCON_ERR_LAUNCH;
        }
        g_addr[dev] = static_cast<float *>(p);
    }
    *out = g_addr[dev];
    return FALCON_OK;
}

}  // namespace

extern "C" int falcon_fwd_masked_noalloc(falcon_variant variant, falcon_dtype dtype,
                                         const void *q, const void *k, const void *v, const void *beta,
                                         const float *lambda, float eps, int window,
                                         int B, int H, int L, int d_k, int d_v,
                                         void *out, float *final_state, cudaStream_t stream) {
    if (variant < FALCON_F1 || variant > FALCON_F3A) return FALCON_ERR_ENUM;
    if (dtype != FALCON_F32 && dtype != FALCON_BF16) return FALCON_ERR_ENUM;
    const bool has_window = variant == FALCON_F3 || variant == FALCON_F3A;
    if (has_window && (window < 1 || window > kMaxWindow)) return FALCON_ERR_WINDOW;
    auto dim_ok = [](int d) { return d == 16 || d == 32 || d == 64 || d == 128; };
    if (B < 0 || H < 0 || L < 0 || !dim_ok(d_k) || !dim_ok(d_v)) return FALCON_ERR_SHAPE;
    FwdParams p{};
    p.variant = variant; p.form = FALCON_MASKED; p.pairing = FALCON_PAIR_PREFIX; p.phi = FALCON_PHI_L2;
    p.window = has_window ? window : 1;
    p.B = B; p.H = H; p.L = L; p.dk = d_k; p.dv = d_v; p.chunk = 64; p.eps = eps;
    p.q = q; p.k = k; p.v = v; p.beta = beta; p.lambda = lambda;
    p.out = out; p.final_state = final_state;
    const size_t nr = masked_ws_r_floats(p), neg = masked_ws_eg_floats(p);
    if (nr + 2 * neg > kNoAllocScratchFloats) return FALCON_ERR_SCRATCH;
    if ((size_t)B * H == 0) return FALCON_OK;
    if (L == 0) {
        if (!final_state) return FALCON_OK;
        const cudaError_t e = cudaMemsetAsync(final_state, 0, sizeof(float) * (size_t)B * H * d_v * d_k, stream);
        return e == cudaSuccess ? FALCON_OK : FALCON_ERR_LAUNCH;
    }
    if (!q || !k || !v || !beta || !lambda || !out) return FALCON_ERR_NULL;
    float *ws = nullptr;
    const int rc = scratch_address(&ws);
    if (rc) return rc;
    p.ws_r = ws;
    p.ws_eta = ws + nr;
    p.ws_gam = p.ws_eta + neg;
    const int lrc = dtype == FALCON_BF16 ? launch_span_masked<__nv_bfloat16>(p, stream)
                                         : launch_span_masked<float>(p, stream);
    if (lrc) return lrc;
    return cudaGetLastError() == cudaSuccess ? FALCON_OK : FALCON_ERR_LAUNCH;
}
