// api.cu -- the C ABI of libfalcon.so (declared in include/falcon.h):
// argument validation, dispatch to the kernels, stream-ordered scratch.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/falcon.h"
#include "common.cuh"
#include "kernels.h"

using namespace falcon;

namespace {

bool dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

int validate_common(int variant, int dtype, int window) {
    if (variant < FALCON_F1 || variant > FALCON_F3A) return FALCON_ERR_ENUM;
    if (dtype != FALCON_F32 && dtype != FALCON_BF16) return FALCON_ERR_ENUM;
    const bool has_window = variant == FALCON_F3 || variant == FALCON_F3A;
    if (has_window && (window < 1 || window > kMaxWindow)) return FALCON_ERR_WINDOW;
    return FALCON_OK;
}

int launched(int rc) {
    if (rc != 0) return rc;
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FALCON_OK : FALCON_ERR_LAUNCH;
}

}  // namespace

namespace falcon {

int validate_fwd(int variant, int form, int dtype, int pairing, int phi, int window, int B, int H, int L, int d_k,
                 int d_v, int chunk) {
    const int rc = validate_common(variant, dtype, window);
    if (rc) return rc;
    if (form < FALCON_RECURRENT || form > FALCON_CHUNK) return FALCON_ERR_ENUM;
    if (pairing != FALCON_PAIR_PREFIX && pairing != FALCON_PAIR_SAME_STEP) return FALCON_ERR_ENUM;
    if (phi != FALCON_PHI_L2 && phi != FALCON_PHI_IDENTITY) return FALCON_ERR_ENUM;
    if (B < 0 || H < 0 || L < 0 || !dim_ok(d_k) || !dim_ok(d_v)) return FALCON_ERR_SHAPE;
    if (form == FALCON_CHUNK && !(chunk == 16 || chunk == 32 || chunk == 64)) return FALCON_ERR_CHUNK;
    return FALCON_OK;
}

}  // namespace falcon

namespace {

int fwd_impl(falcon_variant variant, falcon_form form, falcon_dtype dtype, falcon_pairing pairing, falcon_phi phi,
             const void *q, const void *k, const void *v, const void *beta, const float *lambda, float eps,
             int window, int B, int H, int L, int d_k, int d_v, int chunk, const float *init_state,
             const float *x_prev, const float *win, void *out, float *final_state, cudaStream_t stream) {
    int rc = validate_fwd(variant, form, dtype, pairing, phi, window, B, H, L, d_k, d_v, chunk);
    if (rc) return rc;
    const bool has_window = variant == FALCON_F3 || variant == FALCON_F3A;
    FwdParams p{};
    p.variant = variant; p.form = form; p.pairing = pairing; p.phi = phi;
    p.window = has_window ? window : 1;
    p.B = B; p.H = H; p.L = L; p.dk = d_k; p.dv = d_v; p.chunk = chunk; p.eps = eps;
    p.q = q; p.k = k; p.v = v; p.beta = beta; p.lambda = lambda;
    p.out = out; p.final_state = final_state;
    p.init_state = init_state; p.x_prev = x_prev; p.win = p.window > 1 ? win : nullptr;
    const bool carry = init_state || x_prev || p.win;
    if (carry && form == FALCON_MASKED) return FALCON_ERR_UNSUPPORTED;
    if ((size_t)B * H == 0) return FALCON_OK;
    if (L == 0) {
        if (!final_state) return FALCON_OK;
        cudaError_t e;
        if (init_state)
            e = cudaMemcpyAsync(final_state, init_state, sizeof(float) * (size_t)B * H * d_v * d_k,
                                cudaMemcpyDeviceToDevice, stream);
        else
            e = cudaMemsetAsync(final_state, 0, sizeof(float) * (size_t)B * H * d_v * d_k, stream);
        return e == cudaSuccess ? FALCON_OK : FALCON_ERR_LAUNCH;
    }
    if (!q || !k || !v || !beta || !lambda || !out) return FALCON_ERR_NULL;

    const bool bf16 = dtype == FALCON_BF16;
    if (form == FALCON_RECURRENT)
        return launched(bf16 ? launch_recurrent<__nv_bfloat16>(p, stream) : launch_recurrent<float>(p, stream));
    if (form == FALCON_CHUNK) {
        if (bf16) {
            int tc = launch_split_chunk(p, stream);
            if (tc == 1) tc = launch_pc_chunk(p, stream);
            if (tc == 1) tc = launch_f2_chunk(p, stream);
            if (tc == 1) tc = launch_w_chunk(p, stream);
            if (tc != 1) return launched(tc);  // 1: shape not covered by the tensor-core kernels
        }
        return launched(bf16 ? launch_span_chunk<__nv_bfloat16>(p, stream) : launch_span_chunk<float>(p, stream));
    }
    // masked-parallel: scratch for the solved unknowns, the steps and Gamma
    const size_t nr = masked_ws_r_floats(p), neg = masked_ws_eg_floats(p);
    void *ws = nullptr;
    if (scratch_alloc(&ws, sizeof(float) * (nr + 2 * neg), stream) != cudaSuccess) {
        cudaGetLastError();
        return FALCON_ERR_ALLOC;
    }
    p.ws_r = static_cast<float *>(ws);
    p.ws_eta = p.ws_r + nr;
    p.ws_gam = p.ws_eta + neg;
    rc = launched(bf16 ? launch_span_masked<__nv_bfloat16>(p, stream) : launch_span_masked<float>(p, stream));
    scratch_free(ws, stream);
    return rc;
}

}  // namespace

extern "C" int falcon_fwd_ex(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                             falcon_pairing pairing, falcon_phi phi,
                             const void *q, const void *k, const void *v, const void *beta,
                             const float *lambda, float eps, int window,
                             int B, int H, int L, int d_k, int d_v, int chunk,
                             void *out, float *final_state, cudaStream_t stream) {
    return fwd_impl(variant, form, dtype, pairing, phi, q, k, v, beta, lambda, eps, window, B, H, L, d_k, d_v,
                    chunk, nullptr, nullptr, nullptr, out, final_state, stream);
}

extern "C" int falcon_fwd_carry(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                                const void *q, const void *k, const void *v, const void *beta,
                                const float *lambda, float eps, int window,
                                int B, int H, int L, int d_k, int d_v, int chunk,
                                const float *initial_state, const float *x_prev, const float *win,
                                void *out, float *final_state, cudaStream_t stream) {
    return fwd_impl(variant, form, dtype, FALCON_PAIR_PREFIX, FALCON_PHI_L2, q, k, v, beta, lambda, eps, window,
                    B, H, L, d_k, d_v, chunk, initial_state, x_prev, win, out, final_state, stream);
}

extern "C" int falcon_fwd(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                          const void *q, const void *k, const void *v, const void *beta,
                          const float *lambda, float eps, int window,
                          int B, int H, int L, int d_k, int d_v, int chunk,
                          void *out, float *final_state, cudaStream_t stream) {
    return falcon_fwd_ex(variant, form, dtype, FALCON_PAIR_PREFIX, FALCON_PHI_L2, q, k, v, beta, lambda,
                         eps, window, B, H, L, d_k, d_v, chunk, out, final_state, stream);
}

extern "C" int falcon_decode_step(falcon_variant variant, falcon_dtype dtype,
                                  const void *q, const void *k, const void *v, const void *beta,
                                  const float *lambda, float eps, int window,
                                  int N, int H, int d_k, int d_v,
                                  float *state, float *x_prev, float *win, void *out,
                                  cudaStream_t stream) {
    int rc = validate_common(variant, dtype, window);
    if (rc) return rc;
    if (N < 0 || H < 0 || !dim_ok(d_k) || !dim_ok(d_v)) return FALCON_ERR_SHAPE;
    const bool has_window = variant == FALCON_F3 || variant == FALCON_F3A;
    const int w = has_window ? window : 1;
    if ((size_t)N * H == 0) return FALCON_OK;
    if (!q || !k || !v || !beta || !lambda || !state || !x_prev || !out) return FALCON_ERR_NULL;
    if (w > 1 && !win) return FALCON_ERR_NULL;
    DecodeParams p{};
    p.variant = variant; p.window = w; p.N = N; p.H = H; p.dk = d_k; p.dv = d_v; p.eps = eps;
    p.q = q; p.k = k; p.v = v; p.beta = beta; p.lambda = lambda;
    p.state = state; p.x_prev = x_prev; p.win = w > 1 ? win : nullptr; p.out = out;
    return launched(dtype == FALCON_BF16 ? launch_decode<__nv_bfloat16>(p, stream) : launch_decode<float>(p, stream));
}

extern "C" int falcon_decode_carry_from_prefill(falcon_variant variant, falcon_dtype dtype,
                                                const void *k, const void *v, int window,
                                                int B, int H, int L, int d_k, int d_v,
                                                float *x_prev, float *win, cudaStream_t stream) {
    int rc = validate_common(variant, dtype, window);
    if (rc) return rc;
    if (B < 0 || H < 0 || L < 0 || !dim_ok(d_k) || !dim_ok(d_v)) return FALCON_ERR_SHAPE;
    const bool has_window = variant == FALCON_F3 || variant == FALCON_F3A;
    const int w = has_window ? window : 1;
    if ((size_t)B * H == 0) return FALCON_OK;
    if (!x_prev || (L > 0 && (!k || !v))) return FALCON_ERR_NULL;
    if (w > 1 && !win) return FALCON_ERR_NULL;
    CarryParams p{};
    p.variant = variant; p.window = w; p.B = B; p.H = H; p.L = L; p.dk = d_k; p.dv = d_v;
    p.k = k; p.v = v; p.x_prev = x_prev; p.win = w > 1 ? win : nullptr;
    return launched(dtype == FALCON_BF16 ? launch_carry<__nv_bfloat16>(p, stream) : launch_carry<float>(p, stream));
}

extern "C" int falcon_bwd(falcon_variant variant, falcon_dtype dtype, falcon_pairing pairing, falcon_phi phi,
                          const void *q, const void *k, const void *v, const void *beta, const float *lambda,
                          float eps, int window, int B, int H, int L, int d_k, int d_v, const void *dout,
                          const float *dstate, float *dq, float *dk, float *dv, float *dbeta, float *dlambda,
                          cudaStream_t stream) {
    int rc = validate_common(variant, dtype, window);
    if (rc) return rc;
    if (pairing != FALCON_PAIR_PREFIX && pairing != FALCON_PAIR_SAME_STEP) return FALCON_ERR_ENUM;
    if (phi != FALCON_PHI_L2 && phi != FALCON_PHI_IDENTITY) return FALCON_ERR_ENUM;
    if (B < 0 || H < 0 || L < 0 || !dim_ok(d_k) || !dim_ok(d_v)) return FALCON_ERR_SHAPE;
    if (d_k != d_v || d_k < 32) return FALCON_ERR_UNSUPPORTED;
    const bool has_window = variant == FALCON_F3 || variant == FALCON_F3A;
    if ((size_t)B * H == 0) return FALCON_OK;
    if (L == 0) {
        if (!dlambda) return FALCON_OK;
        return cudaMemsetAsync(dlambda, 0, sizeof(float) * H, stream) == cudaSuccess ? FALCON_OK
                                                                                     : FALCON_ERR_LAUNCH;
    }
    if (!q || !k || !v || !beta || !lambda || !dout || !dq || !dk || !dv || !dbeta) return FALCON_ERR_NULL;
    BwdParams p{};
    p.variant = variant; p.pairing = pairing; p.phi = phi; p.window = has_window ? window : 1;
    p.B = B; p.H = H; p.L = L; p.dk = d_k; p.dv = d_v; p.eps = eps;
    p.q = q; p.k = k; p.v = v; p.beta = beta; p.dout = dout; p.lambda = lambda; p.dstate = dstate;
    p.dq = dq; p.dk_out = dk; p.dv_out = dv; p.dbeta = dbeta; p.dlambda = dlambda;
    return launched(dtype == FALCON_BF16 ? launch_bwd<__nv_bfloat16>(p, stream) : launch_bwd<float>(p, stream));
}

extern "C" int falcon_device_wait_timeouts(unsigned int *count) {
    if (!count) return FALCON_ERR_NULL;
    *count = split_wait_timeouts() + pc_wait_timeouts() + f2_wait_timeouts() + w_wait_timeouts();
    return cudaGetLastError() == cudaSuccess ? FALCON_OK : FALCON_ERR_LAUNCH;
}

extern "C" int falcon_scratch_trim(void) {
    return scratch_trim() == cudaSuccess ? FALCON_OK : FALCON_ERR_LAUNCH;
}

extern "C" const char *falcon_status_string(int status) {
    switch (status) {
        case FALCON_OK: return "ok";
        case FALCON_ERR_NULL: return "a required pointer is NULL";
        case FALCON_ERR_ENUM: return "invalid variant, form, dtype, pairing or feature map";
        case FALCON_ERR_SHAPE: return "unsupported shape: B,H,L must be >= 0 and d_k,d_v in {16,32,64,128}";
        case FALCON_ERR_CHUNK: return "chunk must be 16, 32 or 64 for the chunk-parallel form";
        case FALCON_ERR_WINDOW: return "window must be in [1,8] for Falcon-3/3A";
        case FALCON_ERR_LAUNCH: return "kernel launch failed";
        case FALCON_ERR_ALLOC: return "stream-ordered scratch allocation failed";
        case FALCON_ERR_UNSUPPORTED: return "unsupported combination";
        case FALCON_ERR_SCRATCH: return "problem exceeds the fixed scratch of falcon_fwd_masked_noalloc";
    }
    return "unknown status";
}
