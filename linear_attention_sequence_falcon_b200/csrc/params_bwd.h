// params_bwd.h -- the parameter block of the backward pass (falcon_bwd).
// Not installed; the public boundary is include/falcon.h.
#pragma once

#include <stddef.h>

namespace falcon {

struct BwdParams {
    int variant, pairing, phi, window;
    // form of the forward whose derivative is taken: 0 recurrent, 2 chunk
    // (chunk-parallel backward of Falcon-1/1A, bf16, d = 64, chunk 64)
    int form, chunk, dtype_bf16;
    int B, H, L, dk, dv;
    float eps;
    const void *q, *k, *v, *beta, *dout;
    const float *lambda, *dstate;
    float *dq, *dk_out, *dv_out, *dbeta, *dlambda;
    // the call's workspace (see FwdParams)
    void *ws;
    size_t ws_bytes;
    int ws_given;
};

}  // namespace falcon
