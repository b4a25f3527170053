// api.cu -- the C ABI of libfalcon.so (declared in include/falcon.h):
// argument validation, dispatch to the kernels, stream-ordered scratch.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

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
    if (form == FALCON_CHUNK && !(chunk == 16 || chunk == 32 || chunk == 64)) {
        // chunk 128: the tensor-core path of Falcon-1/1A with bf16 inputs and d_k = d_v <= 64 only
        const bool c128 = chunk == 128 && (variant == FALCON_F1 || variant == FALCON_F1A) &&
                          dtype == FALCON_BF16 && d_k == d_v && (d_k == 32 || d_k == 64);
        if (!c128) return FALCON_ERR_CHUNK;
    }
    return FALCON_OK;
}

}  // namespace falcon

namespace {

// The parameter block of a forward with the arguments' shape (no pointers).
FwdParams shape_params(int variant, int form, int pairing, int phi, int window, int B, int H, int L, int d_k,
                       int d_v, int chunk) {
    const bool has_window = variant == FALCON_F3 || variant == FALCON_F3A;
    FwdParams p{};
    p.variant = variant; p.form = form; p.pairing = pairing; p.phi = phi;
    p.window = has_window ? window : 1;
    p.B = B; p.H = H; p.L = L; p.dk = d_k; p.dv = d_v; p.chunk = chunk;
    return p;
}

// Bytes of workspace the call with these shapes needs: the bf16 tensor-core
// paths that hand per-chunk results between kernels (Falcon-1/1A and
// Falcon-3A at d = 64, Falcon-2A at d = 128, chunk 64) and the
// masked-parallel form; 0 otherwise.
size_t fwd_ws_need(const FwdParams &p, int dtype) {
    if ((size_t)p.B * p.H * p.L == 0) return 0;
    if (p.form == FALCON_MASKED) {
        // the CUDA-core kernel's scratch; the tensor-core kernel (Falcon-1/1A,
        // bf16, d = 64) takes its own, the larger of the two (misaligned
        // pointers send that call to the CUDA-core kernel)
        const size_t span = sizeof(float) * (masked_ws_r_floats(p) + 2 * masked_ws_eg_floats(p));
        return dtype == FALCON_BF16 && masked_tc_covers(p) ? std::max(span, masked_tc_ws_bytes(p)) : span;
    }
    if (p.form != FALCON_CHUNK || dtype != FALCON_BF16) return 0;
    if (split_chunk_covers(p)) return split_chunk_ws_bytes(p);
    if (pc_chunk_covers(p)) return pc_chunk_ws_bytes(p);
    if (w_local_covers(p)) return w_local_ws_bytes(p);
    return 0;
}

int fwd_impl(falcon_variant variant, falcon_form form, falcon_dtype dtype, falcon_pairing pairing, falcon_phi phi,
             const void *q, const void *k, const void *v, const void *beta, const float *lambda, float eps,
             int window, int B, int H, int L, int d_k, int d_v, int chunk, const float *init_state,
             const float *x_prev, const float *win, void *out, float *final_state, int ws_given, void *ws_ptr,
             size_t ws_bytes, cudaStream_t stream) {
    int rc = validate_fwd(variant, form, dtype, pairing, phi, window, B, H, L, d_k, d_v, chunk);
    if (rc) return rc;
    FwdParams p = shape_params(variant, form, pairing, phi, window, B, H, L, d_k, d_v, chunk);
    p.eps = eps;
    p.q = q; p.k = k; p.v = v; p.beta = beta; p.lambda = lambda;
    p.out = out; p.final_state = final_state;
    // under the same-step pair the first sample is phi(k_1) of the segment
    // itself: x_prev is not read
    p.init_state = init_state; p.x_prev = pairing == FALCON_PAIR_PREFIX ? x_prev : nullptr;
    p.win = p.window > 1 ? win : nullptr;
    p.ws = ws_ptr; p.ws_bytes = ws_bytes; p.ws_given = ws_given;
    if (ws_given && fwd_ws_need(p, dtype) > 0 &&
        (!ws_ptr || ws_bytes < fwd_ws_need(p, dtype) || (reinterpret_cast<uintptr_t>(ws_ptr) & 255u) != 0))
        return FALCON_ERR_WORKSPACE;
    const bool carry = init_state || p.x_prev || p.win;
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
            if (tc == 1) tc = launch_seq_chunk(p, stream);
            if (tc == 1) tc = launch_pc_chunk(p, stream);
            if (tc == 1) tc = launch_f2_chunk(p, stream);
            if (tc == 1) tc = launch_w_chunk(p, stream);
            if (tc != 1) return launched(tc);  // 1: shape not covered by the tensor-core kernels
        }
        return launched(bf16 ? launch_span_chunk<__nv_bfloat16>(p, stream) : launch_span_chunk<float>(p, stream));
    }
    // masked-parallel: the tensor-core kernel (Falcon-1/1A, bf16, d = 64), else
    // the CUDA-core kernel with scratch for the solved unknowns, the steps and Gamma
    void *ws = nullptr;
    bool owned = false;
    rc = ws_acquire(ws_given, ws_ptr, ws_bytes, fwd_ws_need(p, dtype), stream, &ws, &owned);
    if (rc) return rc;
    int mrc = bf16 ? launch_masked_tc(p, ws, stream) : 1;
    if (mrc == 1) {
        const size_t nr = masked_ws_r_floats(p), neg = masked_ws_eg_floats(p);
        p.ws_r = static_cast<float *>(ws);
        p.ws_eta = p.ws_r + nr;
        p.ws_gam = p.ws_eta + neg;
        mrc = bf16 ? launch_span_masked<__nv_bfloat16>(p, stream) : launch_span_masked<float>(p, stream);
    }
    rc = launched(mrc);
    ws_release(ws, owned, stream);
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
                    chunk, nullptr, nullptr, nullptr, out, final_state, 0, nullptr, 0, stream);
}

extern "C" int falcon_fwd_carry(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                                const void *q, const void *k, const void *v, const void *beta,
                                const float *lambda, float eps, int window,
                                int B, int H, int L, int d_k, int d_v, int chunk,
                                const float *initial_state, const float *x_prev, const float *win,
                                void *out, float *final_state, cudaStream_t stream) {
    return fwd_impl(variant, form, dtype, FALCON_PAIR_PREFIX, FALCON_PHI_L2, q, k, v, beta, lambda, eps, window,
                    B, H, L, d_k, d_v, chunk, initial_state, x_prev, win, out, final_state, 0, nullptr, 0, stream);
}

extern "C" int falcon_fwd_carry_ex(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                                   falcon_pairing pairing, falcon_phi phi,
                                   const void *q, const void *k, const void *v, const void *beta,
                                   const float *lambda, float eps, int window,
                                   int B, int H, int L, int d_k, int d_v, int chunk,
                                   const float *initial_state, const float *x_prev, const float *win,
                                   void *out, float *final_state, cudaStream_t stream) {
    return fwd_impl(variant, form, dtype, pairing, phi, q, k, v, beta, lambda, eps, window, B, H, L, d_k, d_v,
                    chunk, initial_state, x_prev, win, out, final_state, 0, nullptr, 0, stream);
}

extern "C" int falcon_fwd_workspace_size(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                                         falcon_pairing pairing, falcon_phi phi, int window,
                                         int B, int H, int L, int d_k, int d_v, int chunk, size_t *bytes) {
    if (!bytes) return FALCON_ERR_NULL;
    *bytes = 0;
    const int rc = validate_fwd(variant, form, dtype, pairing, phi, window, B, H, L, d_k, d_v, chunk);
    if (rc) return rc;
    *bytes = fwd_ws_need(shape_params(variant, form, pairing, phi, window, B, H, L, d_k, d_v, chunk), dtype);
    return FALCON_OK;
}

extern "C" int falcon_fwd_ws(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                             falcon_pairing pairing, falcon_phi phi,
                             const void *q, const void *k, const void *v, const void *beta,
                             const float *lambda, float eps, int window,
                             int B, int H, int L, int d_k, int d_v, int chunk,
                             const float *initial_state, const float *x_prev, const float *win,
                             void *out, float *final_state, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
    return fwd_impl(variant, form, dtype, pairing, phi, q, k, v, beta, lambda, eps, window, B, H, L, d_k, d_v,
                    chunk, initial_state, x_prev, win, out, final_state, 1, workspace, workspace_bytes, stream);
}

extern "C" int falcon_fwd(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                          const void *q, const void *k, const void *v, const void *beta,
                          const float *lambda, float eps, int window,
                          int B, int H, int L, int d_k, int d_v, int chunk,
                          void *out, float *final_state, cudaStream_t stream) {
    return falcon_fwd_ex(variant, form, dtype, FALCON_PAIR_PREFIX, FALCON_PHI_L2, q, k, v, beta, lambda,
                         eps, window, B, H, L, d_k, d_v, chunk, out, final_state, stream);
}

namespace {

int decode_impl(falcon_variant variant, falcon_dtype dtype, falcon_pairing pairing, const void *q, const void *k,
                const void *v, const void *beta, const float *lambda, float eps, int window, int N, int H, int d_k,
                int d_v, float *state, float *x_prev, float *win, void *out, cudaStream_t stream) {
    int rc = validate_common(variant, dtype, window);
    if (rc) return rc;
    if (pairing != FALCON_PAIR_PREFIX && pairing != FALCON_PAIR_SAME_STEP) return FALCON_ERR_ENUM;
    if (N < 0 || H < 0 || !dim_ok(d_k) || !dim_ok(d_v)) return FALCON_ERR_SHAPE;
    const bool has_window = variant == FALCON_F3 || variant == FALCON_F3A;
    const int w = has_window ? window : 1;
    if ((size_t)N * H == 0) return FALCON_OK;
    if (!q || !k || !v || !beta || !lambda || !state || !out) return FALCON_ERR_NULL;
    // the prefix pair's sample is the carried x_prev; the same-step pair's is phi(k_t)
    if (pairing == FALCON_PAIR_PREFIX && !x_prev) return FALCON_ERR_NULL;
    if (w > 1 && !win) return FALCON_ERR_NULL;
    DecodeParams p{};
    p.variant = variant; p.window = w; p.pairing = pairing; p.N = N; p.H = H; p.dk = d_k; p.dv = d_v; p.eps = eps;
    p.q = q; p.k = k; p.v = v; p.beta = beta; p.lambda = lambda;
    p.state = state; p.x_prev = x_prev; p.win = w > 1 ? win : nullptr; p.out = out;
    return launched(dtype == FALCON_BF16 ? launch_decode<__nv_bfloat16>(p, stream) : launch_decode<float>(p, stream));
}

int carry_impl(falcon_variant variant, falcon_dtype dtype, falcon_pairing pairing, const void *k, const void *v,
               int window, int B, int H, int L, int d_k, int d_v, float *x_prev, float *win, cudaStream_t stream) {
    int rc = validate_common(variant, dtype, window);
    if (rc) return rc;
    if (pairing != FALCON_PAIR_PREFIX && pairing != FALCON_PAIR_SAME_STEP) return FALCON_ERR_ENUM;
    if (B < 0 || H < 0 || L < 0 || !dim_ok(d_k) || !dim_ok(d_v)) return FALCON_ERR_SHAPE;
    const bool has_window = variant == FALCON_F3 || variant == FALCON_F3A;
    const int w = has_window ? window : 1;
    if ((size_t)B * H == 0) return FALCON_OK;
    if (L > 0 && (!k || !v)) return FALCON_ERR_NULL;
    if (pairing == FALCON_PAIR_PREFIX && !x_prev) return FALCON_ERR_NULL;
    if (w > 1 && !win) return FALCON_ERR_NULL;
    if (!x_prev && w == 1) return FALCON_OK;  // same-step pair, no window: nothing to carry
    CarryParams p{};
    p.variant = variant; p.window = w; p.pairing = pairing; p.B = B; p.H = H; p.L = L; p.dk = d_k; p.dv = d_v;
    p.k = k; p.v = v; p.x_prev = x_prev; p.win = w > 1 ? win : nullptr;
    return launched(dtype == FALCON_BF16 ? launch_carry<__nv_bfloat16>(p, stream) : launch_carry<float>(p, stream));
}

int bwd_impl(falcon_variant variant, falcon_form form, falcon_dtype dtype, falcon_pairing pairing, falcon_phi phi,
             const void *q, const void *k, const void *v, const void *beta, const float *lambda, float eps,
             int window, int B, int H, int L, int d_k, int d_v, int chunk, const void *dout, const float *dstate,
             float *dq, float *dk, float *dv, float *dbeta, float *dlambda, int ws_given, void *ws_ptr,
             size_t ws_bytes, cudaStream_t stream, size_t *need_only) {
    int rc = validate_common(variant, dtype, window);
    if (rc) return rc;
    if (pairing != FALCON_PAIR_PREFIX && pairing != FALCON_PAIR_SAME_STEP) return FALCON_ERR_ENUM;
    if (phi != FALCON_PHI_L2 && phi != FALCON_PHI_IDENTITY) return FALCON_ERR_ENUM;
    if (form != FALCON_RECURRENT && form != FALCON_CHUNK) return form == FALCON_MASKED ? FALCON_ERR_UNSUPPORTED
                                                                                     : FALCON_ERR_ENUM;
    if (B < 0 || H < 0 || L < 0 || !dim_ok(d_k) || !dim_ok(d_v)) return FALCON_ERR_SHAPE;
    if (d_k != d_v || d_k < 32) return FALCON_ERR_UNSUPPORTED;
    if (form == FALCON_CHUNK) {
        if (chunk != 64) return FALCON_ERR_CHUNK;
        if (!(variant == FALCON_F1 || variant == FALCON_F1A) || dtype != FALCON_BF16 || d_k != 64)
            return FALCON_ERR_UNSUPPORTED;
    }
    const bool has_window = variant == FALCON_F3 || variant == FALCON_F3A;
    BwdParams p{};
    p.variant = variant; p.pairing = pairing; p.phi = phi; p.window = has_window ? window : 1;
    p.form = form; p.chunk = chunk; p.dtype_bf16 = dtype == FALCON_BF16;
    p.B = B; p.H = H; p.L = L; p.dk = d_k; p.dv = d_v; p.eps = eps;
    if (need_only) {
        *need_only = bwd_ws_bytes(p);
        return FALCON_OK;
    }
    if (ws_given && bwd_ws_bytes(p) > 0 &&
        (!ws_ptr || ws_bytes < bwd_ws_bytes(p) || (reinterpret_cast<uintptr_t>(ws_ptr) & 255u) != 0))
        return FALCON_ERR_WORKSPACE;
    if ((size_t)B * H == 0) return FALCON_OK;
    if (L == 0) {
        if (!dlambda) return FALCON_OK;
        return cudaMemsetAsync(dlambda, 0, sizeof(float) * H, stream) == cudaSuccess ? FALCON_OK
                                                                                     : FALCON_ERR_LAUNCH;
    }
    if (!q || !k || !v || !beta || !lambda || !dout || !dq || !dk || !dv || !dbeta) return FALCON_ERR_NULL;
    p.q = q; p.k = k; p.v = v; p.beta = beta; p.dout = dout; p.lambda = lambda; p.dstate = dstate;
    p.dq = dq; p.dk_out = dk; p.dv_out = dv; p.dbeta = dbeta; p.dlambda = dlambda;
    p.ws = ws_ptr; p.ws_bytes = ws_bytes; p.ws_given = ws_given;
    return launched(dtype == FALCON_BF16 ? launch_bwd<__nv_bfloat16>(p, stream) : launch_bwd<float>(p, stream));
}

}  // namespace

extern "C" int falcon_decode_step(falcon_variant variant, falcon_dtype dtype,
                                  const void *q, const void *k, const void *v, const void *beta,
                                  const float *lambda, float eps, int window,
                                  int N, int H, int d_k, int d_v,
                                  float *state, float *x_prev, float *win, void *out,
                                  cudaStream_t stream) {
    return decode_impl(variant, dtype, FALCON_PAIR_PREFIX, q, k, v, beta, lambda, eps, window, N, H, d_k, d_v,
                       state, x_prev, win, out, stream);
}

extern "C" int falcon_decode_step_ex(falcon_variant variant, falcon_dtype dtype, falcon_pairing pairing,
                                     const void *q, const void *k, const void *v, const void *beta,
                                     const float *lambda, float eps, int window,
                                     int N, int H, int d_k, int d_v,
                                     float *state, float *x_prev, float *win, void *out,
                                     cudaStream_t stream) {
    return decode_impl(variant, dtype, pairing, q, k, v, beta, lambda, eps, window, N, H, d_k, d_v, state, x_prev,
                       win, out, stream);
}

extern "C" int falcon_decode_carry_from_prefill(falcon_variant variant, falcon_dtype dtype,
                                                const void *k, const void *v, int window,
                                                int B, int H, int L, int d_k, int d_v,
                                                float *x_prev, float *win, cudaStream_t stream) {
    return carry_impl(variant, dtype, FALCON_PAIR_PREFIX, k, v, window, B, H, L, d_k, d_v, x_prev, win, stream);
}

extern "C" int falcon_decode_carry_from_prefill_ex(falcon_variant variant, falcon_dtype dtype,
                                                   falcon_pairing pairing, const void *k, const void *v, int window,
                                                   int B, int H, int L, int d_k, int d_v,
                                                   float *x_prev, float *win, cudaStream_t stream) {
    return carry_impl(variant, dtype, pairing, k, v, window, B, H, L, d_k, d_v, x_prev, win, stream);
}

extern "C" int falcon_bwd(falcon_variant variant, falcon_dtype dtype, falcon_pairing pairing, falcon_phi phi,
                          const void *q, const void *k, const void *v, const void *beta, const float *lambda,
                          float eps, int window, int B, int H, int L, int d_k, int d_v, const void *dout,
                          const float *dstate, float *dq, float *dk, float *dv, float *dbeta, float *dlambda,
                          cudaStream_t stream) {
    return bwd_impl(variant, FALCON_RECURRENT, dtype, pairing, phi, q, k, v, beta, lambda, eps, window, B, H, L,
                    d_k, d_v, 64, dout, dstate, dq, dk, dv, dbeta, dlambda, 0, nullptr, 0, stream, nullptr);
}

extern "C" int falcon_bwd_ex(falcon_variant variant, falcon_form form, falcon_dtype dtype, falcon_pairing pairing,
                             falcon_phi phi, const void *q, const void *k, const void *v, const void *beta,
                             const float *lambda, float eps, int window, int B, int H, int L, int d_k, int d_v,
                             int chunk, const void *dout, const float *dstate, float *dq, float *dk, float *dv,
                             float *dbeta, float *dlambda, cudaStream_t stream) {
    return bwd_impl(variant, form, dtype, pairing, phi, q, k, v, beta, lambda, eps, window, B, H, L, d_k, d_v,
                    chunk, dout, dstate, dq, dk, dv, dbeta, dlambda, 0, nullptr, 0, stream, nullptr);
}

extern "C" int falcon_bwd_workspace_size(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                                         falcon_pairing pairing, falcon_phi phi, int window, int B, int H, int L,
                                         int d_k, int d_v, int chunk, size_t *bytes) {
    if (!bytes) return FALCON_ERR_NULL;
    *bytes = 0;
    return bwd_impl(variant, form, dtype, pairing, phi, nullptr, nullptr, nullptr, nullptr, nullptr, 0.f, window, B,
                    H, L, d_k, d_v, chunk, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 0,
                    nullptr, 0, 0, bytes);
}

extern "C" int falcon_bwd_ws(falcon_variant variant, falcon_form form, falcon_dtype dtype, falcon_pairing pairing,
                             falcon_phi phi, const void *q, const void *k, const void *v, const void *beta,
                             const float *lambda, float eps, int window, int B, int H, int L, int d_k, int d_v,
                             int chunk, const void *dout, const float *dstate, float *dq, float *dk, float *dv,
                             float *dbeta, float *dlambda, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
    return bwd_impl(variant, form, dtype, pairing, phi, q, k, v, beta, lambda, eps, window, B, H, L, d_k, d_v,
                    chunk, dout, dstate, dq, dk, dv, dbeta, dlambda, 1, workspace, workspace_bytes, stream,
                    nullptr);
}

extern "C" int falcon_device_wait_timeouts(unsigned int *count) {
    if (!count) return FALCON_ERR_NULL;
    *count = split_wait_timeouts() + pc_wait_timeouts() + f2_wait_timeouts() + w_wait_timeouts() +
             masked_wait_timeouts() + decode_wait_timeouts();
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
        case FALCON_ERR_CHUNK:
            return "chunk must be 16, 32 or 64 for the chunk-parallel form (128: Falcon-1/1A, bf16, d = 32 or 64)";
        case FALCON_ERR_WINDOW: return "window must be in [1,8] for Falcon-3/3A";
        case FALCON_ERR_LAUNCH: return "kernel launch failed";
        case FALCON_ERR_ALLOC: return "stream-ordered scratch allocation failed";
        case FALCON_ERR_UNSUPPORTED: return "unsupported combination";
        case FALCON_ERR_SCRATCH: return "problem exceeds the fixed scratch of falcon_fwd_masked_noalloc";
        case FALCON_ERR_WORKSPACE:
            return "the caller's workspace is missing, smaller than the size query gave or not 256-byte aligned";
    }
    return "unknown status";
}
