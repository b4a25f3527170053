// k_bwd.cu -- backward pass of Falcon-1/2 and Falcon-1A/2A (one sample per
// update) in the recurrent form, fp32 on the CUDA cores: the gradients of a
// loss with respect to q, k, v, beta and lambda, given dL/do (and dL/dS_L).
// The inner-product family is described first; the regression family's sweep
// (bwd_sweep_reg_kernel) follows it.
//
// The chunk form trains on the recurrent function (page "Fast Weight
// Attention：用于持续学习的快速权重注意力", 核心方法 3); its derivative, with
// S_t = alpha_t o S_{t-1} + (eta_t o y_t) x_t^T (per value channel j for
// Falcon-2A; page "借鉴40年前的设想！…", 02 (2)) and o_t = S_t q_t:
//   dq_t = S_t^T do_t,
//   Gs_t = dL/dS_t = do_t q_t^T + alpha_{t+1} o Gs_{t+1}   (Gs_L = dL/dS_L),
//   dy_t = eta_t o (Gs_t x_t),  deta_t = y_t o (Gs_t x_t),  dx_t = Gs_t^T (eta_t o y_t).
// The decays need no stored past state: with G_t = sum_{r<=t} log alpha_r,
//   dL/dG_t = do_t o o_t - (eta_t o y_t) o (Gs_t x_t)      (per channel),
// plus <dL/dS_L, S_L> (per row) at the last token, whose G the final state
// carries as well,
//   dL/dlog alpha_t = sum_{t'>=t} dL/dG_t',
// then alpha = max(1 - eta lambda, 2^-20) (no gradient on the floor), eta =
// beta / (eps + |x|^2) (0 at x = 0) and x = k / |k| (or k) take it to beta,
// lambda and k.
//
// Four kernels: per-token samples and steps (a warp per token), the two
// sweeps per head (a block per (b, h); S, then Gs, in shared memory; tokens
// staged 32 at a time), the decay chain (a block-wide reverse scan per (b, h,
// channel)) and a warp per token for the feature map.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace falcon {

namespace {

constexpr int TT = 32;  // tokens staged per tile

template <typename T>
__device__ __forceinline__ float ld(const T *p, size_t i) {
    return to_f32(p[i]);
}

// per token: x_t (fp32), |x_t|^2, eta_t, alpha_t; a warp per (b, h, t)
template <typename T>
__global__ void __launch_bounds__(256) bwd_prep_kernel(BwdParams p, float *xs, float *ns, float *etas, float *alphas) {
    const size_t gw = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const size_t rows = (size_t)p.B * p.H * p.L;
    if (gw >= rows) return;
    const int D = p.dk, t = (int)(gw % p.L);
    const size_t bh = gw / p.L;
    const int kr = p.pairing == 0 ? t - 1 : t;
    const T *k = static_cast<const T *>(p.k) + bh * (size_t)p.L * D;
    float ss = 0.f;
    for (int c = lane; c < D; c += 32) {
        const float v = kr >= 0 ? ld(k, (size_t)kr * D + c) : 0.f;
        ss += v * v;
    }
    ss = group_sum<32>(ss);
    const float inv = p.phi != 0 ? 1.f : (ss > 0.f ? rsqrtf(ss) : 0.f);
    for (int c = lane; c < D; c += 32) xs[gw * D + c] = kr >= 0 ? ld(k, (size_t)kr * D + c) * inv : 0.f;
    const float n = ss * inv * inv;
    if (lane == 0) ns[gw] = n;
    const int nch = (p.variant == F2A || p.variant == F2) ? p.dv : 1;
    const float lam = p.lambda[bh % p.H];
    const T *beta = static_cast<const T *>(p.beta) + bh * (size_t)p.L * nch;
    for (int ch = lane; ch < nch; ch += 32) {
        float eta, alpha;
        step_and_decay(ld(beta, (size_t)t * nch + ch), n, p.eps, lam, eta, alpha);
        etas[gw * nch + ch] = eta;
        alphas[gw * nch + ch] = alpha;
    }
}

// The two sweeps of one (b, h).  S (then Gs) in shared memory, D x (D+1).
template <typename T, int D>
__global__ void __launch_bounds__(256, 1) bwd_sweep_kernel(BwdParams p, const float *xs, const float *etas,
                                                          const float *alphas, float *dga, float *dgb, float *deta,
                                                          float *dx) {
    constexpr int NT = 256, LD = D + 1, RPT = NT / D, SEG = D / RPT;
    extern __shared__ float sm[];
    float *S = sm;                                  // [D][LD]
    float *tq = S + D * LD, *tdo = tq + TT * D;     // [TT][D] staged q, do
    float *ty = tdo + TT * D, *tx = ty + TT * D;    // staged y, x
    float *te = tx + TT * D, *ta = te + TT * D;     // staged eta, alpha (per channel; scalars repeat)
    float *ta_next = ta + TT * D;                   // alpha of the token after the tile ([D])
    const int tid = threadIdx.x, L = p.L;
    const size_t bh = blockIdx.x;
    const int nch = (p.variant == F2A || p.variant == F2) ? D : 1;
    const T *q = static_cast<const T *>(p.q) + bh * (size_t)L * D;
    const T *v = static_cast<const T *>(p.v) + bh * (size_t)L * D;
    const T *dout = static_cast<const T *>(p.dout) + bh * (size_t)L * D;
    const float *x = xs + bh * (size_t)L * D;
    const float *et = etas + bh * (size_t)L * nch, *al = alphas + bh * (size_t)L * nch;
    float *dq = p.dq + bh * (size_t)L * D, *dv = p.dv_out + bh * (size_t)L * D;
    float *ga = dga + bh * (size_t)L * nch, *gb = dgb + bh * (size_t)L * nch, *de = deta + bh * (size_t)L * nch;
    float *dxo = dx + bh * (size_t)L * D;

    auto stage = [&](int t0, int n) {
        for (int e = tid; e < TT * D; e += NT) {
            const int i = e / D, c = e % D, t = t0 + i;
            const bool in = i < n;
            tq[e] = in ? ld(q, (size_t)t * D + c) : 0.f;
            tdo[e] = in ? ld(dout, (size_t)t * D + c) : 0.f;
            ty[e] = in ? ld(v, (size_t)t * D + c) : 0.f;
            tx[e] = in ? x[(size_t)t * D + c] : 0.f;
            te[e] = in ? et[(size_t)t * nch + (nch > 1 ? c : 0)] : 0.f;
            ta[e] = in ? al[(size_t)t * nch + (nch > 1 ? c : 0)] : 1.f;
        }
    };
    // row / column of this thread in the reductions
    const int rj = tid / RPT, rp = tid % RPT;

    // ---- forward sweep: S_t, then dq_t = S_t^T do_t and do_t o o_t
    for (int e = tid; e < D * LD; e += NT) S[e] = 0.f;
    for (int t0 = 0; t0 < L; t0 += TT) {
        const int n = min(TT, L - t0);
        __syncthreads();
        stage(t0, n);
        __syncthreads();
        for (int i = 0; i < n; ++i) {
            const int t = t0 + i;
            for (int e = tid; e < D * D; e += NT) {
                const int j = e / D, c = e % D;
                S[j * LD + c] = ta[i * D + j] * S[j * LD + c] + te[i * D + j] * ty[i * D + j] * tx[i * D + c];
            }
            __syncthreads();
            float o = 0.f, g = 0.f, f = 0.f;  // row rj: (S q)_j; column rj: (S^T do)_c
#pragma unroll 8
            for (int s = 0; s < SEG; ++s) {
                const int c = rp * SEG + s;
                o = fmaf(S[rj * LD + c], tq[i * D + c], o);
                g = fmaf(S[c * LD + rj], tdo[i * D + c], g);
            }
            // the final state is e^{G_{L-1}} (...) too: dL/dG_{L-1} also takes <dS_L, S_L> (row rj)
            if (t == L - 1 && p.dstate) {
                for (int s = 0; s < SEG; ++s) {
                    const int c = rp * SEG + s;
                    f = fmaf(S[rj * LD + c], p.dstate[(bh * D + rj) * D + c], f);
                }
            }
#pragma unroll
            for (int o2 = RPT / 2; o2 > 0; o2 >>= 1) {
                o += __shfl_xor_sync(0xffffffffu, o, o2);
                g += __shfl_xor_sync(0xffffffffu, g, o2);
                f += __shfl_xor_sync(0xffffffffu, f, o2);
            }
            if (rp == 0) {
                dq[(size_t)t * D + rj] = g;
                const float a = tdo[i * D + rj] * o + f;
                if (nch > 1) ga[(size_t)t * D + rj] = a;
                else tx[i * D + rj] = a;  // x of this token is no longer needed: reuse it
            }
            __syncthreads();
            if (nch == 1 && tid < 32) {
                float a = 0.f;
                for (int j = tid; j < D; j += 32) a += tx[i * D + j];
                a = group_sum<32>(a);
                if (tid == 0) ga[t] = a;
            }
        }
    }
    // ---- reverse sweep: Gs_t, dy_t, deta_t, dx_t and (eta y) o (Gs x)
    __syncthreads();
    for (int e = tid; e < D * D; e += NT) {
        const int j = e / D, c = e % D;
        S[j * LD + c] = p.dstate ? p.dstate[(bh * D + j) * D + c] : 0.f;
    }
    for (int e = tid; e < D; e += NT) ta_next[e] = 1.f;  // no step after the last token
    const int ntile = (L + TT - 1) / TT;
    for (int tb = ntile - 1; tb >= 0; --tb) {
        const int t0 = tb * TT, n = min(TT, L - t0);
        __syncthreads();
        stage(t0, n);
        __syncthreads();
        for (int i = n - 1; i >= 0; --i) {
            const int t = t0 + i;
            const float *anext = i + 1 < n ? ta + (i + 1) * D : ta_next;
            for (int e = tid; e < D * D; e += NT) {
                const int j = e / D, c = e % D;
                S[j * LD + c] = anext[j] * S[j * LD + c] + tdo[i * D + j] * tq[i * D + c];
            }
            __syncthreads();
            float gx = 0.f, dxc = 0.f;  // row rj: (Gs x)_j; column rj: (Gs^T (eta o y))_c
#pragma unroll 8
            for (int s = 0; s < SEG; ++s) {
                const int c = rp * SEG + s;
                gx = fmaf(S[rj * LD + c], tx[i * D + c], gx);
                dxc = fmaf(S[c * LD + rj], te[i * D + c] * ty[i * D + c], dxc);
            }
#pragma unroll
            for (int o2 = RPT / 2; o2 > 0; o2 >>= 1) {
                gx += __shfl_xor_sync(0xffffffffu, gx, o2);
                dxc += __shfl_xor_sync(0xffffffffu, dxc, o2);
            }
            if (rp == 0) {
                const float eta = te[i * D + rj], y = ty[i * D + rj];
                dv[(size_t)t * D + rj] = eta * gx;
                dxo[(size_t)t * D + rj] = dxc;
                if (nch > 1) {
                    de[(size_t)t * D + rj] = y * gx;
                    gb[(size_t)t * D + rj] = eta * y * gx;
                } else {
                    tdo[i * D + rj] = y * gx;  // do of this token is no longer needed: reuse it
                }
            }
            __syncthreads();
            if (nch == 1 && tid < 32) {
                float a = 0.f;
                for (int j = tid; j < D; j += 32) a += tdo[i * D + j];
                a = group_sum<32>(a);
                if (tid == 0) {
                    de[t] = a;
                    gb[t] = te[i * D] * a;
                }
            }
        }
        __syncthreads();
        for (int e = tid; e < D; e += NT) ta_next[e] = ta[e];  // alpha of this tile's first token
    }
}

// The regression family (Falcon-1 / Falcon-2): S_t = alpha_t S_{t-1} +
// eta_t (y_t - S_{t-1} x_t) x_t^T.  Its derivative needs S_{t-1} at every
// step of the reverse sweep: the forward sweep keeps S at the start of every
// tile of TT tokens (ck), and the reverse sweep recomputes a tile's states
// from its checkpoint (ts, global scratch of the block) before walking it
// backwards.  Per step, with Gs = dL/dS_t (do_t q_t^T added):
//   e = y - S_{t-1} x,  de = eta (Gs x),  dalpha = <Gs, S_{t-1}> (per row),
//   deta = e . (Gs x) (per row),  dy = de,
//   dx = Gs^T (eta o e) - S_{t-1}^T de,  Gs <- alpha o Gs - de x^T.
// dalpha is written straight into dga (the scan is not needed here).
template <typename T, int D>
__global__ void __launch_bounds__(256, 1) bwd_sweep_reg_kernel(BwdParams p, const float *xs, const float *etas,
                                                              const float *alphas, float *dga, float *deta, float *dx,
                                                              float *ck, float *ts) {
    constexpr int NT = 256, LD = D + 1, RPT = NT / D, SEG = D / RPT;
    extern __shared__ float sm[];
    float *S = sm;                                  // [D][LD]: S, then Gs
    float *tq = S + D * LD, *tdo = tq + TT * D;
    float *ty = tdo + TT * D, *tx = ty + TT * D;
    float *te = tx + TT * D, *ta = te + TT * D;
    float *ve = ta + TT * D, *vde = ve + D;         // [D] e_j and de_j of the current step
    float *vsum = vde + D;                          // [3 * D] row sums for the Falcon-1 totals
    const int tid = threadIdx.x, L = p.L;
    const size_t bh = blockIdx.x;
    const int nch = p.variant == F2 ? D : 1;
    const T *q = static_cast<const T *>(p.q) + bh * (size_t)L * D;
    const T *v = static_cast<const T *>(p.v) + bh * (size_t)L * D;
    const T *dout = static_cast<const T *>(p.dout) + bh * (size_t)L * D;
    const float *x = xs + bh * (size_t)L * D;
    const float *et = etas + bh * (size_t)L * nch, *al = alphas + bh * (size_t)L * nch;
    float *dq = p.dq + bh * (size_t)L * D, *dv = p.dv_out + bh * (size_t)L * D;
    float *ga = dga + bh * (size_t)L * nch, *de = deta + bh * (size_t)L * nch;
    float *dxo = dx + bh * (size_t)L * D;
    const int ntile = (L + TT - 1) / TT;
    float *cks = ck + bh * (size_t)ntile * D * D;   // S before each tile
    float *tss = ts + bh * (size_t)TT * D * D;      // S before each token of the tile being walked

    auto stage = [&](int t0, int n) {
        for (int e = tid; e < TT * D; e += NT) {
            const int i = e / D, c = e % D, t = t0 + i;
            const bool in = i < n;
            tq[e] = in ? ld(q, (size_t)t * D + c) : 0.f;
            tdo[e] = in ? ld(dout, (size_t)t * D + c) : 0.f;
            ty[e] = in ? ld(v, (size_t)t * D + c) : 0.f;
            tx[e] = in ? x[(size_t)t * D + c] : 0.f;
            te[e] = in ? et[(size_t)t * nch + (nch > 1 ? c : 0)] : 0.f;
            ta[e] = in ? al[(size_t)t * nch + (nch > 1 ? c : 0)] : 1.f;
        }
    };
    const int rj = tid / RPT, rp = tid % RPT;
    // one regression step on the state in S with token i of the staged tile
    auto step = [&](int i) {
        float r = 0.f;  // (S x)_rj
#pragma unroll 8
        for (int s = 0; s < SEG; ++s) {
            const int c = rp * SEG + s;
            r = fmaf(S[rj * LD + c], tx[i * D + c], r);
        }
#pragma unroll
        for (int o2 = RPT / 2; o2 > 0; o2 >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o2);
        if (rp == 0) ve[rj] = ty[i * D + rj] - r;
        __syncthreads();
        for (int e = tid; e < D * D; e += NT) {
            const int j = e / D, c = e % D;
            S[j * LD + c] = ta[i * D + j] * S[j * LD + c] + te[i * D + j] * ve[j] * tx[i * D + c];
        }
        __syncthreads();
    };

    // ---- forward sweep: checkpoints, S_t, dq_t = S_t^T do_t
    for (int e = tid; e < D * LD; e += NT) S[e] = 0.f;
    for (int tb = 0; tb < ntile; ++tb) {
        const int t0 = tb * TT, n = min(TT, L - t0);
        __syncthreads();
        stage(t0, n);
        for (int e = tid; e < D * D; e += NT) cks[(size_t)tb * D * D + e] = S[(e / D) * LD + e % D];
        __syncthreads();
        for (int i = 0; i < n; ++i) {
            step(i);
            float g = 0.f;
#pragma unroll 8
            for (int s = 0; s < SEG; ++s) {
                const int c = rp * SEG + s;
                g = fmaf(S[c * LD + rj], tdo[i * D + c], g);
            }
#pragma unroll
            for (int o2 = RPT / 2; o2 > 0; o2 >>= 1) g += __shfl_xor_sync(0xffffffffu, g, o2);
            if (rp == 0) dq[(size_t)(t0 + i) * D + rj] = g;
        }
    }
    // ---- reverse sweep, tile by tile; Gs = dL/dS in S between tiles
    __syncthreads();
    for (int e = tid; e < D * D; e += NT) {
        const int j = e / D, c = e % D;
        S[j * LD + c] = p.dstate ? p.dstate[(bh * D + j) * D + c] : 0.f;  // dL/dS_L
    }
    for (int tb = ntile - 1; tb >= 0; --tb) {
        const int t0 = tb * TT, n = min(TT, L - t0);
        float *ckt = cks + (size_t)tb * D * D;
        __syncthreads();
        stage(t0, n);
        // swap Gs and the tile's checkpoint (each element by one thread)
        for (int e = tid; e < D * D; e += NT) {
            const int j = e / D, c = e % D;
            const float sv = ckt[e];
            ckt[e] = S[j * LD + c];
            S[j * LD + c] = sv;
        }
        __syncthreads();
        // recompute the tile: tss[i] = S before token t0 + i
        for (int i = 0; i < n; ++i) {
            for (int e = tid; e < D * D; e += NT) tss[(size_t)i * D * D + e] = S[(e / D) * LD + e % D];
            step(i);
        }
        for (int e = tid; e < D * D; e += NT) S[(e / D) * LD + e % D] = ckt[e];
        __syncthreads();
        for (int i = n - 1; i >= 0; --i) {
            const int t = t0 + i;
            const float *Sp = tss + (size_t)i * D * D;
            for (int e = tid; e < D * D; e += NT) {
                const int j = e / D, c = e % D;
                S[j * LD + c] += tdo[i * D + j] * tq[i * D + c];
            }
            __syncthreads();
            float sx = 0.f, gx = 0.f, gs = 0.f;  // row rj: (S_{t-1} x), (Gs x), <Gs, S_{t-1}>
#pragma unroll 8
            for (int s2 = 0; s2 < SEG; ++s2) {
                const int c = rp * SEG + s2;
                const float sp = Sp[(size_t)rj * D + c], g = S[rj * LD + c];
                sx = fmaf(sp, tx[i * D + c], sx);
                gx = fmaf(g, tx[i * D + c], gx);
                gs = fmaf(g, sp, gs);
            }
#pragma unroll
            for (int o2 = RPT / 2; o2 > 0; o2 >>= 1) {
                sx += __shfl_xor_sync(0xffffffffu, sx, o2);
                gx += __shfl_xor_sync(0xffffffffu, gx, o2);
                gs += __shfl_xor_sync(0xffffffffu, gs, o2);
            }
            if (rp == 0) {
                const float eta = te[i * D + rj], e = ty[i * D + rj] - sx, d = eta * gx;
                ve[rj] = eta * e;
                vde[rj] = d;
                dv[(size_t)t * D + rj] = d;
                if (nch > 1) {
                    ga[(size_t)t * D + rj] = gs;
                    de[(size_t)t * D + rj] = e * gx;
                } else {
                    vsum[rj] = gs;
                    vsum[D + rj] = e * gx;
                }
            }
            __syncthreads();
            float dxc = 0.f;  // column rj: sum_j (eta e)_j Gs[j][c] - de_j S_{t-1}[j][c]
#pragma unroll 8
            for (int s2 = 0; s2 < SEG; ++s2) {
                const int j = rp * SEG + s2;
                dxc = fmaf(ve[j], S[j * LD + rj], dxc);
                dxc = fmaf(-vde[j], Sp[(size_t)j * D + rj], dxc);
            }
#pragma unroll
            for (int o2 = RPT / 2; o2 > 0; o2 >>= 1) dxc += __shfl_xor_sync(0xffffffffu, dxc, o2);
            if (rp == 0) dxo[(size_t)t * D + rj] = dxc;
            if (nch == 1 && tid < 32) {
                float a = 0.f, b = 0.f;
                for (int j = tid; j < D; j += 32) {
                    a += vsum[j];
                    b += vsum[D + j];
                }
                a = group_sum<32>(a);
                b = group_sum<32>(b);
                if (tid == 0) {
                    ga[t] = a;
                    de[t] = b;
                }
            }
            __syncthreads();
            // Gs <- alpha o Gs - de x^T (dL/dS_{t-1})
            for (int e = tid; e < D * D; e += NT) {
                const int j = e / D, c = e % D;
                S[j * LD + c] = ta[i * D + j] * S[j * LD + c] - vde[j] * tx[i * D + c];
            }
            __syncthreads();
        }
    }
}

// decay chain: one block per (b, h, channel).  dlog alpha_t = sum_{t'>=t}
// (ga - gb)_t' as a block-wide reverse scan over tiles of 2048 tokens (eight
// per thread, latest tile first, the sum of the later tiles carried), then
// alpha and eta per token; writes dbeta, each channel's share of dL/d|x|^2
// (over deta) and dlambda.
template <typename T>
__global__ void __launch_bounds__(256) bwd_decay_kernel(BwdParams p, const float *ns, const float *etas,
                                                       const float *alphas, const float *dga, const float *dgb,
                                                       float *deta) {
    constexpr int PER = 8, TS = 256 * PER;
    __shared__ float wsum[8];
    __shared__ float wlam[8];
    const int nch = (p.variant == F2A || p.variant == F2) ? p.dv : 1;
    const size_t bh = blockIdx.x / nch;
    const int ch = (int)(blockIdx.x % nch), L = p.L, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool reg = p.variant == F1 || p.variant == F2;
    const float lam = p.lambda[bh % p.H];
    const T *beta = static_cast<const T *>(p.beta) + bh * (size_t)L * nch;
    float carry = 0.f, dlam = 0.f;
    for (int t1 = L; t1 > 0; t1 -= TS) {
        const int t0 = max(0, t1 - TS), base = t0 + tid * PER;
        float v[PER], sfx[PER];
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int t = base + k;
            const size_t i = (bh * L + t) * nch + ch;
            v[k] = (t < t1 && !reg) ? dga[i] - dgb[i] : 0.f;
        }
        float run = 0.f;
#pragma unroll
        for (int k = PER - 1; k >= 0; --k) {
            run += v[k];
            sfx[k] = run;  // sum over this thread's tokens >= base + k
        }
        // suffix sums over the later threads of the warp, then over the later warps
        float x = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, x, o);
            if (lane + o < 32) x += y;
        }
        if (lane == 0) wsum[warp] = x;
        __syncthreads();
        float later = x - run;
        float tile = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            if (w > warp) later += wsum[w];
            tile += wsum[w];
        }
        later += carry;
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int t = base + k;
            if (t >= t1) continue;
            const size_t i = (bh * L + t) * nch + ch;
            const float a = alphas[i], eta = etas[i], n = ns[bh * L + t];
            // the regression family's sweep gives dL/dalpha directly
            const float dalpha = reg ? dga[i] : (sfx[k] + later) / a;
            float d = deta[i];
            if (1.f - eta * lam > kAlphaFloor) {
                d -= lam * dalpha;
                dlam -= eta * dalpha;
            }
            p.dbeta[i] = n > 0.f ? d / (p.eps + n) : 0.f;
            deta[i] = n > 0.f ? -d * ld(beta, (size_t)t * nch + ch) / ((p.eps + n) * (p.eps + n)) : 0.f;
        }
        carry += tile;
        __syncthreads();
    }
    dlam = group_sum<32>(dlam);
    if (lane == 0) wlam[warp] = dlam;
    __syncthreads();
    if (tid == 0 && p.dlambda) {
        float s = 0.f;
        for (int w = 0; w < 8; ++w) s += wlam[w];
        atomicAdd(&p.dlambda[bh % p.H], s);
    }
}

// a warp per (b, h, t): dx_t += 2 dn_t x_t, then dk of the key x_t came from
template <typename T>
__global__ void __launch_bounds__(256) bwd_key_kernel(BwdParams p, const float *xs, const float *dnc, const float *dx) {
    const size_t gw = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= (size_t)p.B * p.H * p.L) return;
    const int D = p.dk, L = p.L, t = (int)(gw % L);
    const size_t bh = gw / L;
    const int nch = (p.variant == F2A || p.variant == F2) ? p.dv : 1;
    float dn = 0.f;
    for (int ch = lane; ch < nch; ch += 32) dn += dnc[gw * nch + ch];
    dn = group_sum<32>(dn);
    // the key row this token's sample was made from; under the prefix pair the
    // last key feeds no sample and the first sample is zero
    const int kr = p.pairing == 0 ? t - 1 : t;
    float *dkrow = p.dk_out + bh * (size_t)L * D;
    if (p.pairing == 0 && t == L - 1)
        for (int c = lane; c < D; c += 32) dkrow[(size_t)t * D + c] = 0.f;
    if (kr < 0) return;
    const T *k = static_cast<const T *>(p.k) + bh * (size_t)L * D;
    float g[4], xv[4], kk = 0.f, xd = 0.f;  // D <= 128: four per lane
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const int c = lane + 32 * s;
        const bool in = c < D;
        xv[s] = in ? xs[gw * D + c] : 0.f;
        g[s] = in ? dx[gw * D + c] + 2.f * dn * xv[s] : 0.f;
        const float kv = in ? ld(k, (size_t)kr * D + c) : 0.f;
        kk += kv * kv;
        xd += xv[s] * g[s];
    }
    kk = group_sum<32>(kk);
    xd = group_sum<32>(xd);
    const float inv = p.phi != 0 ? 1.f : (kk > 0.f ? rsqrtf(kk) : 0.f);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const int c = lane + 32 * s;
        if (c < D) dkrow[(size_t)kr * D + c] = p.phi != 0 ? g[s] : (g[s] - xv[s] * xd) * inv;
    }
}

template <typename T, int D>
int launch_sweep(const BwdParams &p, const float *xs, const float *etas, const float *alphas, float *dga, float *dgb,
                 float *deta, float *dx, float *ck, float *ts, cudaStream_t s) {
    if (p.variant == F1 || p.variant == F2) {
        const size_t bytes = ((size_t)D * (D + 1) + 6 * TT * D + 5 * D) * sizeof(float);
        cudaFuncSetAttribute(bwd_sweep_reg_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        bwd_sweep_reg_kernel<T, D><<<(unsigned)(p.B * p.H), 256, bytes, s>>>(p, xs, etas, alphas, dga, deta, dx, ck, ts);
        return 0;
    }
    const size_t bytes = ((size_t)D * (D + 1) + 6 * TT * D + D) * sizeof(float);
    cudaFuncSetAttribute(bwd_sweep_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    bwd_sweep_kernel<T, D><<<(unsigned)(p.B * p.H), 256, bytes, s>>>(p, xs, etas, alphas, dga, dgb, deta, dx);
    return 0;
}

}  // namespace

template <typename T>
int launch_bwd(const BwdParams &p, cudaStream_t s) {
    const int D = p.dk, nch = (p.variant == F2A || p.variant == F2) ? D : 1;
    const bool reg = p.variant == F1 || p.variant == F2;
    const size_t rows = (size_t)p.B * p.H * p.L;
    if (rows == 0) return 0;
    // scratch: x, |x|^2, eta, alpha, the two decay-gradient halves, deta, dx;
    // the regression family adds the tile checkpoints and one tile of states per head
    const size_t BH = (size_t)p.B * p.H, ntile = (p.L + TT - 1) / TT;
    const size_t nreg = reg ? BH * (ntile + TT) * D * D : 0;
    const size_t nf = rows * D * 2 + rows + rows * nch * 5 + nreg;
    void *ws = nullptr;
    if (scratch_alloc(&ws, nf * sizeof(float), s) != cudaSuccess) {
        cudaGetLastError();
        return -8;  // FALCON_ERR_ALLOC
    }
    float *xs = static_cast<float *>(ws), *dx = xs + rows * D, *ns = dx + rows * D;
    float *etas = ns + rows, *alphas = etas + rows * nch, *dga = alphas + rows * nch, *dgb = dga + rows * nch;
    float *deta = dgb + rows * nch;
    float *ck = deta + rows * nch, *ts = ck + BH * ntile * D * D;
    const unsigned wblocks = (unsigned)((rows * 32 + 255) / 256);
    bwd_prep_kernel<T><<<wblocks, 256, 0, s>>>(p, xs, ns, etas, alphas);
    int rc = D == 32 ? launch_sweep<T, 32>(p, xs, etas, alphas, dga, dgb, deta, dx, ck, ts, s)
           : D == 64 ? launch_sweep<T, 64>(p, xs, etas, alphas, dga, dgb, deta, dx, ck, ts, s)
                     : launch_sweep<T, 128>(p, xs, etas, alphas, dga, dgb, deta, dx, ck, ts, s);
    const size_t chans = (size_t)p.B * p.H * nch;
    if (p.dlambda) cudaMemsetAsync(p.dlambda, 0, sizeof(float) * p.H, s);
    bwd_decay_kernel<T><<<(unsigned)chans, 256, 0, s>>>(p, ns, etas, alphas, dga, dgb, deta);
    bwd_key_kernel<T><<<wblocks, 256, 0, s>>>(p, xs, deta, dx);
    const cudaError_t e = cudaGetLastError();
    scratch_free(ws, s);
    if (rc != 0) return rc;
    return e == cudaSuccess ? 0 : -7;  // FALCON_ERR_LAUNCH
}

template int launch_bwd<float>(const BwdParams &, cudaStream_t);
template int launch_bwd<__nv_bfloat16>(const BwdParams &, cudaStream_t);

}  // namespace falcon
