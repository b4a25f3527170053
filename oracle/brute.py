"""Unrolled brute force for tiny inputs -- TEST INFRASTRUCTURE.

An independent re-derivation of the Falcon updates written as products of
per-step transition matrices instead of a recurrence, for L <= 16 and small d.
Every Falcon update is affine in S (right-multiplication form):

    S_t = S_{t-1} M_t + b_t,
    M_t = alpha_t I - eta_t sum_{i in W_t} x_i x_i^T   (regression family)
    M_t = alpha_t I                                    (inner-product family)
    b_t = eta_t sum_{i in W_t} y_i x_i^T

([EXPL] 核心方法 1: S_t = S_{t-1} - eta_t grad L with grad (S x - y) x^T or
-y x^T; [NEWS] 02 (1): the old state decays by (1 - eta lambda)).  With S_0 = 0
the state is therefore the sum over writes s of b_s carried forward by the
ordered product M_{s+1} ... M_t, which is what this module evaluates, fresh for
every (s, t) pair, row by row (Falcon-2/2A have one eta, alpha per value
channel j, i.e. per row of S).  Output o_t = S_t q_t.
"""
from __future__ import annotations

import numpy as np

ALPHA_FLOOR = 2.0 ** -20


def _samples(k, pairing, phi):
    L, dk = k.shape
    if phi == "l2":
        nrm = np.sqrt((k * k).sum(-1, keepdims=True))
        f = np.where(nrm > 0, k / np.where(nrm > 0, nrm, 1.0), 0.0)
    else:
        f = k.copy()
    if pairing == "same_step":
        return f
    x = np.zeros_like(f)
    x[1:] = f[:-1]          # x_t = phi(k_{t-1}), x_1 = 0
    return x


def unit(variant, q, k, v, beta, lam, eps, window=1, pairing="prefix", phi="l2", S0=None, x_prev=None,
         carry=None):
    """One (b,h) unit: q,k [L,dk], v [L,dv], beta [L] or [L,dv], lam scalar.
    A segment continuing a sequence starts from S0 [dv,dk] with x_1 = x_prev
    [dk] (prefix pair) and, for Falcon-3/3A, the earlier samples `carry`
    [Bw-1, dk+dv] (x then y, oldest first): then
        S_t = S0 M_1 ... M_t + sum_s b_s M_{s+1} ... M_t.
    Returns (out [L,dv], S_L [dv,dk])."""
    q, k, v, beta = (np.asarray(a, dtype=np.float64) for a in (q, k, v, beta))
    L, dk = q.shape
    dv = v.shape[1]
    reg = variant in ("F1", "F2", "F3")
    w = window if variant in ("F3", "F3A") else 1
    x = _samples(k, pairing, phi)
    if x_prev is not None:
        x[0] = np.asarray(x_prev, dtype=np.float64)
    # samples before the segment: index -m is row P - m of the carry (P = w - 1)
    P = w - 1
    xc = np.zeros((P, dk))
    yc = np.zeros((P, dv))
    if carry is not None and P > 0:
        carry = np.asarray(carry, dtype=np.float64)
        xc, yc = carry[:, :dk], carry[:, dk:]
    x = np.concatenate([xc, x])
    v = np.concatenate([yc, v])
    win = [list(range(t - w + 1 + P, t + 1 + P)) for t in range(L)]
    energy = np.array([sum(float(x[i] @ x[i]) for i in win[t]) for t in range(L)])
    b2 = beta.reshape(L, -1)
    eta = np.where(energy[:, None] > 0, b2 / (eps + energy[:, None]), 0.0)
    eta = np.broadcast_to(eta, (L, dv)) if eta.shape[1] == 1 else eta
    alpha = np.maximum(1.0 - eta * lam, ALPHA_FLOOR)
    eye = np.eye(dk)

    def M(r, j):
        G = sum(np.outer(x[i], x[i]) for i in win[r]) if reg else 0.0
        return alpha[r, j] * eye - eta[r, j] * G

    def bvec(s, j):
        return eta[s, j] * sum(v[i, j] * x[i] for i in win[s])

    S0 = np.zeros((dv, dk)) if S0 is None else np.asarray(S0, dtype=np.float64)
    out = np.zeros((L, dv))
    S = np.zeros((dv, dk))
    for j in range(dv):
        for t in range(L):
            P0 = eye.copy()
            for r in range(t + 1):
                P0 = P0 @ M(r, j)
            row = S0[j] @ P0
            for s in range(t + 1):
                P = eye.copy()
                for r in range(s + 1, t + 1):
                    P = P @ M(r, j)
                row = row + bvec(s, j) @ P
            out[t, j] = row @ q[t]
            if t == L - 1:
                S[j] = row
    return out, S


def fwd(variant, q, k, v, beta, lam, eps, window=1, pairing="prefix", phi="l2"):
    """Batched wrapper over (b,h): shapes as the oracle's fwd."""
    q = np.asarray(q, dtype=np.float64)
    B, H, L, dk = q.shape
    dv = np.asarray(v).shape[-1]
    out = np.zeros((B, H, L, dv))
    S = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            out[b, h], S[b, h] = unit(variant, q[b, h], k[b, h], v[b, h], beta[b, h],
                                      float(np.asarray(lam)[h]), eps, window, pairing, phi)
    return out, S
