"""Pins of the oracle's backward pass (reverse mode of the recurrent
definition), independent of how it is computed:

* central finite differences of the fp64 forward oracle for every input
  (q, k, v, beta, lambda), every variant, both pairings, both feature maps,
  and a case where alpha sits on its floor (no gradient through the clamp);
* closed forms of Falcon-1A without forgetting (lambda = 0, alpha = 1):
  o_t = sum_{s<=t} eta_s (x_s . q_t) y_s and S_L = sum_s eta_s y_s x_s^T, so
  dL/dv_s = eta_s (sum_{t>=s} (x_s . q_t) do_t + dS_L x_s) and
  dL/dq_t = sum_{s<=t} eta_s x_s (y_s . do_t).
"""
import zlib

import numpy as np
import pytest

import oracle

VARIANTS = ("F1", "F2", "F3", "F1A", "F2A", "F3A")


def draw(variant, rng, B=1, H=2, L=7, dk=3, dv=2, lam=0.3, beta_scale=1.0):
    nch = dv if variant in ("F2", "F2A") else 1
    q = rng.standard_normal((B, H, L, dk))
    k = rng.standard_normal((B, H, L, dk))
    v = rng.standard_normal((B, H, L, dv))
    bshape = (B, H, L) if nch == 1 else (B, H, L, dv)
    beta = beta_scale / (1.0 + np.exp(-rng.standard_normal(bshape)))
    return q, k, v, beta, np.full(H, lam)


def numeric_grads(variant, q, k, v, beta, lam, eps, do, dS, **kw):
    def loss(**a):
        o, S = oracle.fwd(variant, "recurrent", a["q"], a["k"], a["v"], a["beta"], a["lam"], eps, **kw)
        return (o * do).sum() + (S * dS).sum()

    base = dict(q=q, k=k, v=v, beta=beta, lam=lam)
    out = {}
    for name in base:
        arr = base[name]
        g = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            h = 1e-6
            a = arr.copy()
            a[idx] += h
            lp = loss(**{**base, name: a})
            a[idx] -= 2 * h
            lm = loss(**{**base, name: a})
            g[idx] = (lp - lm) / (2 * h)
        out[name] = g
    return out


KEYS = {"q": "dq", "k": "dk", "v": "dv", "beta": "dbeta", "lam": "dlambda"}


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("pairing,phi,lam,beta_scale", [
    ("prefix", "l2", 0.3, 1.0),
    ("same_step", "identity", 0.3, 1.0),
    ("prefix", "identity", 0.05, 1.0),
    ("prefix", "l2", 0.9, 2.5),  # alpha = max(1 - eta lambda, 2^-20) on its floor for most tokens
])
def test_backward_matches_finite_differences(variant, pairing, phi, lam, beta_scale):
    rng = np.random.default_rng(zlib.crc32(("%s %s %s %g" % (variant, pairing, phi, lam)).encode()))
    w = 3 if variant in ("F3", "F3A") else 1
    q, k, v, beta, lamv = draw(variant, rng, lam=lam, beta_scale=beta_scale)
    eps = 1e-6
    do = rng.standard_normal(v.shape)
    dS = rng.standard_normal((q.shape[0], q.shape[1], v.shape[-1], q.shape[-1]))
    g = oracle.bwd(variant, q, k, v, beta, lamv, eps, do, dS, window=w, pairing=pairing, phi=phi)
    num = numeric_grads(variant, q, k, v, beta, lamv, eps, do, dS, window=w, pairing=pairing, phi=phi)
    for name, key in KEYS.items():
        ref = num[name]
        err = np.abs(ref - g[key]).max() / max(np.abs(ref).max(), 1e-12)
        assert err < 1e-6, (name, err)


def test_backward_closed_form_without_forgetting():
    rng = np.random.default_rng(7)
    B, H, L, dk, dv = 2, 2, 9, 4, 3
    q, k, v, beta, _ = draw("F1A", rng, B, H, L, dk, dv)
    lam = np.zeros(H)
    eps = 1e-6
    do = rng.standard_normal(v.shape)
    dS = rng.standard_normal((B, H, dv, dk))
    g = oracle.bwd("F1A", q, k, v, beta, lam, eps, do, dS)
    # samples and steps written out: x_t = k_{t-1}/|k_{t-1}|, x_0 = 0, eta = beta/(eps + |x|^2)
    x = np.zeros_like(k)
    x[:, :, 1:] = k[:, :, :-1] / np.linalg.norm(k[:, :, :-1], axis=-1, keepdims=True)
    n = (x * x).sum(-1)
    eta = np.where(n > 0, beta / (eps + n), 0.0)
    for b in range(B):
        for h in range(H):
            X, Q, Y, E, D = x[b, h], q[b, h], v[b, h], eta[b, h], do[b, h]
            xq = X @ Q.T  # [s, t] = x_s . q_t
            dv_ref = np.zeros((L, dv))
            dq_ref = np.zeros((L, dk))
            for s in range(L):
                dv_ref[s] = E[s] * (sum(xq[s, t] * D[t] for t in range(s, L)) + dS[b, h] @ X[s])
            for t in range(L):
                dq_ref[t] = sum(E[s] * X[s] * (Y[s] @ D[t]) for s in range(t + 1))
            assert np.abs(g["dv"][b, h] - dv_ref).max() < 1e-12
            assert np.abs(g["dq"][b, h] - dq_ref).max() < 1e-12
    assert np.abs(g["dlambda"]).max() > 0  # lambda = 0 is not clamped: its gradient is -sum eta dalpha


def test_dlambda_term_mass():
    """dlambda_l1 is the mass of the terms dlambda sums: |dlambda| <= mass,
    with equality for a single token (one term), and the mass of a batch is
    the sum of its rows' masses."""
    rng = np.random.default_rng(7)
    q, k, v, beta, lam = draw("F1", rng, L=40, B=3)
    do = rng.standard_normal(v.shape)
    g = oracle.bwd("F1", q, k, v, beta, lam, 1e-6, do)
    assert np.all(np.abs(g["dlambda"]) <= g["dlambda_l1"] + 1e-12) and np.all(g["dlambda_l1"] > 0)
    parts = [oracle.bwd("F1", q[b:b + 1], k[b:b + 1], v[b:b + 1], beta[b:b + 1], lam, 1e-6, do[b:b + 1])
             for b in range(3)]
    np.testing.assert_allclose(sum(p["dlambda_l1"] for p in parts), g["dlambda_l1"], rtol=1e-12)
    # two tokens under the prefix pair: x_1 = 0, so only token 2 steps: one term
    q2, k2, v2, b2, l2 = (a[:1, :, :2] if a.ndim > 1 else a for a in (q, k, v, beta, lam))
    g2 = oracle.bwd("F1", q2, k2, v2, b2, lam, 1e-6, do[:1, :, :2])
    np.testing.assert_allclose(np.abs(g2["dlambda"]), g2["dlambda_l1"], rtol=1e-12)


def test_backward_of_an_empty_sequence():
    rng = np.random.default_rng(3)
    q, k, v, beta, lam = draw("F2A", rng, L=0)
    g = oracle.bwd("F2A", q, k, v, beta, lam, 1e-6, np.zeros(v.shape))
    assert all(a.size == 0 for key, a in g.items() if key not in ("dlambda", "dlambda_l1"))
    assert np.all(g["dlambda"] == 0) and np.all(g["dlambda_l1"] == 0)
