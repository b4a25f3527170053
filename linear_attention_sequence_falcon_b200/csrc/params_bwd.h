// params_bwd.h -- the parameter block of the backward pass (falcon_bwd).
// Not installed; the public boundary is include/falcon.h.
#pragma once

namespace falcon {

struct BwdParams {
    int variant, pairing, phi, window;
    int B, H, L, dk, dv;
    float eps;
    const void *q, *k, *v, *beta, *dout;
    const float *lambda, *dstate;
    float *dq, *dk_out, *dv_out, *dbeta, *dlambda;
};

}  // namespace falcon
