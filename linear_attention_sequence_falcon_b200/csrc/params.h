// params.h -- the parameter blocks the C ABI (api.cu) hands to the kernels.
// Not installed; the public boundary is include/falcon.h.
#pragma once

#include <stddef.h>

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
    // the call's workspace: the caller's block (ws_given, ws_bytes long) or,
    // when not given, stream-ordered memory drawn by the launcher itself
    void *ws;
    size_t ws_bytes;
    int ws_given;
    // optional: the state entering every chunk, [B,H,nchunks,dv,dk] fp32
    // (written by the Falcon-1/1A tensor-core path for the chunk-parallel
    // backward)
    float *states_out;
};

struct DecodeParams {
    int variant, window, pairing;
    int N, H, dk, dv;
    float eps;
    const void *q, *k, *v, *beta;
    const float *lambda;
    float *state, *x_prev, *win;
    void *out;
};

struct CarryParams {
    int variant, window, pairing;
    int B, H, L, dk, dv;
    const void *k, *v;
    float *x_prev, *win;
};

}  // namespace falcon
