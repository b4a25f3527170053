// params.h -- the parameter blocks the C ABI (api.cu) hands to the kernels.
// Not installed; the public boundary is include/falcon.h.
#pragma once

namespace falcon {

struct FwdParams {
    int variant, form, pairing, phi, window;
    int B, H, L, dk, dv, chunk;
    float eps;
    const void *q, *k, *v, *beta;
    const float *lambda;
    void *out;
    float *final_state;
    // stream-ordered scratch for the masked-parallel form
    float *ws_r, *ws_eta, *ws_gam;
    // a segment continuing a sequence (NULL: zeros, the start of a sequence):
    // initial state [B,H,dv,dk], x_prev [B,H,dk] (x of the first token) and
    // the window-1 samples before the segment [B,H,window-1,dk+dv]
    const float *init_state, *x_prev, *win;
};

struct DecodeParams {
    int variant, window;
    int N, H, dk, dv;
    float eps;
    const void *q, *k, *v, *beta;
    const float *lambda;
    float *state, *x_prev, *win;
    void *out;
};

struct CarryParams {
    int variant, window;
    int B, H, L, dk, dv;
    const void *k, *v;
    float *x_prev, *win;
};

}  // namespace falcon
