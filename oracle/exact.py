"""Exact rational arithmetic statement of the Falcon recurrence -- TEST INFRASTRUCTURE.

Used only to write the small fixtures under tests/golden/ (by the script there)
so that the fp64 oracle can be held to values with no rounding at all.  Inputs
are Fractions; the L2 feature map needs keys whose norms are rational (e.g.
(3,4)/5), which the fixture script chooses; anything else raises.

Update ([EXPL] 核心方法 1 and 2; [NEWS] 02 (1) and (2)):
  x_t = phi(k_{t-1}) (prefix pair, x_1 = 0) or phi(k_t) (same-step pair)
  eta_t = beta_t / (eps + n_t), n_t = |x_t|^2 (window energy for Falcon-3/3A),
          eta_t = 0 when n_t = 0
  alpha_t = max(1 - eta_t lambda, 2^-20)
  regression:    S_t = alpha S_{t-1} + eta sum_{i in W_t} (y_i - S_{t-1} x_i) x_i^T
  inner product: S_t = alpha S_{t-1} + eta sum_{i in W_t} y_i x_i^T
  o_t = S_t q_t
"""
from __future__ import annotations

from fractions import Fraction as Fr
from math import isqrt

ALPHA_FLOOR = Fr(1, 2 ** 20)


def _sqrt_exact(a: Fr) -> Fr:
    n, d = a.numerator, a.denominator
    rn, rd = isqrt(n), isqrt(d)
    if rn * rn != n or rd * rd != d:
        raise ValueError("norm is not rational: %s" % a)
    return Fr(rn, rd)


def _phi(k, phi):
    if phi == "identity":
        return list(k)
    n2 = sum(c * c for c in k)
    if n2 == 0:
        return [Fr(0)] * len(k)
    nrm = _sqrt_exact(n2)
    return [c / nrm for c in k]


def unit(variant, q, k, v, beta, lam, eps, window=1, pairing="prefix", phi="l2"):
    """q,k: L lists of dk Fractions; v: L lists of dv; beta: L scalars or L
    lists of dv (Falcon-2/2A); lam, eps: Fractions.  Returns (out, S)."""
    L = len(q)
    dk, dv = len(q[0]), len(v[0])
    reg = variant in ("F1", "F2", "F3")
    w = window if variant in ("F3", "F3A") else 1
    if pairing == "same_step":
        x = [_phi(k[t], phi) for t in range(L)]
    else:
        x = [[Fr(0)] * dk] + [_phi(k[t - 1], phi) for t in range(1, L)]
    S = [[Fr(0)] * dk for _ in range(dv)]
    out = []
    for t in range(L):
        W = list(range(max(0, t - w + 1), t + 1))
        n = sum(sum(c * c for c in x[i]) for i in W)
        res = {}
        for i in W:
            res[i] = [v[i][j] - (sum(S[j][c] * x[i][c] for c in range(dk)) if reg else 0)
                      for j in range(dv)]
        newS = []
        for j in range(dv):
            b = beta[t][j] if isinstance(beta[t], (list, tuple)) else beta[t]
            eta = b / (eps + n) if n > 0 else Fr(0)
            a = max(1 - eta * lam, ALPHA_FLOOR)
            newS.append([a * S[j][c] + eta * sum(res[i][j] * x[i][c] for i in W) for c in range(dk)])
        S = newS
        out.append([sum(S[j][c] * q[t][c] for c in range(dk)) for j in range(dv)])
    return out, S
