"""CPU pins for the fp64 oracle: each test ties it to something other than
itself -- an exact rational evaluation, a textbook special case the pages
name, a closed form of the printed update, or an independent brute force.

Pages cited (title, section):
  [EXPL] "Fast Weight Attention：用于持续学习的快速权重注意力", 核心方法 1-4
  [SUMM] "Fast Weight Attention for Continual Learning", 方法
  [NEWS] "借鉴40年前的设想！字节Seed提出快速权重注意力推进大模型持续学习", 02
"""
import json
import os
from fractions import Fraction as Fr

import numpy as np
import pytest

from oracle import brute

VARIANTS = ("F1", "F2", "F3", "F1A", "F2A", "F3A")
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "exact_small.json")


def rnd(seed, B, H, L, dk, dv, variant, lam_hi=0.05, key_scale=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, L, dk))
    k = rng.standard_normal((B, H, L, dk)) * key_scale
    v = rng.standard_normal((B, H, L, dv))
    bshape = (B, H, L, dv) if variant in ("F2", "F2A") else (B, H, L)
    beta = 1 / (1 + np.exp(-rng.standard_normal(bshape)))
    lam = rng.uniform(0, lam_hi, H)
    return q, k, v, beta, lam


def wnd(variant):
    return 3 if variant in ("F3", "F3A") else 1


# ---------------------------------------------------------------- exact fixtures

def _fr(a):
    if isinstance(a, list):
        return np.array([_fr(x) for x in a], dtype=np.float64)
    return float(Fr(a))


@pytest.mark.parametrize("form", ["recurrent", "masked", "chunk"])
def test_exact_rational_fixtures(oracle_mod, form):
    """fp64 oracle == exact rational evaluation of the printed update
    ([EXPL] 核心方法 1-2, [NEWS] 02 (1)-(2)), every variant, both pairings, both
    feature maps, the positive-decay floor."""
    doc = json.load(open(GOLDEN))
    assert len(doc["cases"]) >= 19
    for c in doc["cases"]:
        q, k, v = (_fr(c[n])[None, None] for n in ("q", "k", "v"))
        beta = _fr(c["beta"])[None, None]
        out, S = oracle_mod.fwd(c["variant"], form, q, k, v, beta, [float(Fr(c["lam"]))],
                                float(Fr(c["eps"])), window=c["window"], chunk=2,
                                pairing=c["pairing"], phi=c["phi"])
        want_o, want_S = _fr(c["out"]), _fr(c["final_state"])
        scale = max(1.0, np.abs(want_o).max())
        assert np.abs(out[0, 0] - want_o).max() <= 1e-12 * scale, c["name"]
        assert np.abs(S[0, 0] - want_S).max() <= 1e-12 * max(1.0, np.abs(want_S).max()), c["name"]


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("pairing,phi", [("prefix", "l2"), ("same_step", "l2"), ("prefix", "identity")])
def test_brute_force_all_forms_all_chunks(oracle_mod, variant, pairing, phi):
    """Unrolled transition-matrix products == every oracle form, every chunk
    size, L <= 16 ("three equivalent implementations", [SUMM] 计算形式与数值稳定)."""
    L, dk, dv = 13, 4, 3
    q, k, v, beta, lam = rnd(7, 1, 2, L, dk, dv, variant, lam_hi=0.3)
    w = wnd(variant)
    eps = 1e-3 if phi == "identity" else 1e-6
    bo, bS = brute.fwd(variant, q, k, v, beta, lam, eps, w, pairing, phi)
    assert np.abs(bo).max() > 1e-3
    runs = [("recurrent", 1), ("masked", 1)] + [("chunk", c) for c in (1, 2, 3, 4, 5, 8, 13, 16)]
    for form, C in runs:
        o, S = oracle_mod.fwd(variant, form, q, k, v, beta, lam, eps, window=w, chunk=C,
                              pairing=pairing, phi=phi)
        np.testing.assert_allclose(o, bo, rtol=1e-9, atol=1e-10, err_msg=f"{form} C={C}")
        np.testing.assert_allclose(S, bS, rtol=1e-9, atol=1e-10, err_msg=f"{form} C={C}")


@pytest.mark.parametrize("variant", VARIANTS)
def test_form_equivalence_medium(oracle_mod, variant):
    """recurrent == masked == chunk at a size the brute force cannot reach,
    with L not a multiple of the chunk (ragged tail)."""
    L, dk, dv = 77, 16, 8
    q, k, v, beta, lam = rnd(11, 2, 2, L, dk, dv, variant)
    w = 4 if variant in ("F3", "F3A") else 1
    o_r, S_r = oracle_mod.fwd(variant, "recurrent", q, k, v, beta, lam, 1e-6, window=w)
    assert np.abs(o_r).max() > 1e-2
    for form, C in (("masked", 1), ("chunk", 16), ("chunk", 32), ("chunk", 64)):
        o, S = oracle_mod.fwd(variant, form, q, k, v, beta, lam, 1e-6, window=w, chunk=C)
        np.testing.assert_allclose(o, o_r, rtol=1e-9, atol=1e-10, err_msg=f"{form} C={C}")
        np.testing.assert_allclose(S, S_r, rtol=1e-9, atol=1e-10, err_msg=f"{form} C={C}")


# ---------------------------------------------------------------- NLMS

def _prefix_states(oracle_mod, variant, q, k, v, beta, lam, eps, phi="l2", window=1):
    """S_t for t = 1..L from runs on each prefix (causality: the final state of
    the length-t prefix is S_t)."""
    L = q.shape[2]
    return [oracle_mod.fwd(variant, "recurrent", q[:, :, :t], k[:, :, :t], v[:, :, :t],
                           beta[:, :, :t], lam, eps, window=window, phi=phi)[1][0, 0]
            for t in range(1, L + 1)]


def test_nlms_reduction_textbook_filter(oracle_mod):
    """lambda=0, eps=0: Falcon-1 is classic NLMS ([NEWS] 02 (1) "exactly reduces to
    classic NLMS"; [EXPL] 核心方法 2, NLMS note).  Checked three ways against the
    adaptive-filter statement, per output channel j with weight w_j, input
    u = k_{t-1} and desired signal d = v_t:
      (a) the textbook filter w <- w + mu e u / |u|^2, e = d - w.u;
      (b) the a-posteriori error equals (1 - mu) times the a-priori error;
      (c) the weight change is the minimum-norm one: it lies along u."""
    L, dk, dv = 12, 5, 3
    q, k, v, beta, lam = rnd(3, 1, 1, L, dk, dv, "F1")
    lam = np.zeros(1)
    S = _prefix_states(oracle_mod, "F1", q, k, v, beta, lam, 0.0, phi="identity")
    # (a) textbook NLMS filter bank
    Wt = np.zeros((dv, dk))
    for t in range(L):
        if t >= 1:
            u = k[0, 0, t - 1]
            mu = beta[0, 0, t]
            for j in range(dv):
                e = v[0, 0, t, j] - Wt[j] @ u
                Wt[j] = Wt[j] + mu * e * u / (u @ u)
        np.testing.assert_allclose(S[t], Wt, rtol=1e-11, atol=1e-12)
    # (b), (c)
    for t in range(1, L):
        u = k[0, 0, t - 1]
        mu = beta[0, 0, t]
        e_prior = v[0, 0, t] - S[t - 1] @ u
        e_post = v[0, 0, t] - S[t] @ u
        np.testing.assert_allclose(e_post, (1 - mu) * e_prior, rtol=1e-10, atol=1e-12)
        dS = S[t] - S[t - 1]
        proj_out = dS - np.outer(dS @ u, u) / (u @ u)
        assert np.abs(proj_out).max() < 1e-12


def test_interpolation_closed_form(oracle_mod):
    """lambda=0, beta=1, eps=0 and unit inputs: each regression step makes the
    new state reproduce its target exactly, S_t x_t = y_t (the update of
    [EXPL] 核心方法 1 with eta = 1/|x|^2)."""
    L, dk, dv = 10, 6, 4
    q, k, v, beta, lam = rnd(5, 1, 1, L, dk, dv, "F1")
    beta = np.ones_like(beta)
    S = _prefix_states(oracle_mod, "F1", q, k, v, beta, np.zeros(1), 0.0)
    for t in range(1, L):
        x = k[0, 0, t - 1] / np.linalg.norm(k[0, 0, t - 1])
        np.testing.assert_allclose(S[t] @ x, v[0, 0, t], rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- linear attention

def _phi(k):
    return k / np.linalg.norm(k, axis=-1, keepdims=True)


@pytest.mark.parametrize("lam", [0.0, 0.07])
def test_linear_attention_reduction(oracle_mod, lam):
    """Inner-product family + same-step pair reduces to causal linear attention
    (lambda=0) and to scalar-decay (Mamba-2-like) accumulation (lambda>0)
    ([NEWS] 02 (2), last list; [EXPL] 核心方法 1 warning paragraph):
      O = ((Q Phi(K)^T) o D) V,  D[t,s] = (1-lambda)^(t-s) for s <= t."""
    L, dk, dv = 40, 8, 5
    q, k, v, beta, _ = rnd(9, 1, 1, L, dk, dv, "F1A")
    beta = np.ones_like(beta)
    out, _ = oracle_mod.fwd("F1A", "recurrent", q, k, v, beta, [lam], 0.0, pairing="same_step")
    Q, K, V = q[0, 0], _phi(k[0, 0]), v[0, 0]
    t = np.arange(L)
    D = np.where(t[:, None] >= t[None, :], (1 - lam) ** (t[:, None] - t[None, :]).clip(0), 0.0)
    want = ((Q @ K.T) * D) @ V
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-11, atol=1e-11)


def test_prefix_pair_is_shifted_linear_attention(oracle_mod):
    """With the prefix-aligned pair (x_t, y_t) = (phi(k_{t-1}), v_t)
    ([SUMM] 输入与状态定义; [EXPL] 核心方法 1) the same reduction pairs v_t with
    the previous key: o_t = sum_{2<=s<=t} (phi(k_{s-1}).q_t) v_s."""
    L, dk, dv = 30, 8, 5
    q, k, v, beta, _ = rnd(13, 1, 1, L, dk, dv, "F1A")
    beta = np.ones_like(beta)
    out, _ = oracle_mod.fwd("F1A", "recurrent", q, k, v, beta, [0.0], 0.0)
    Q, K, V = q[0, 0], _phi(k[0, 0]), v[0, 0]
    want = np.zeros((L, dv))
    for t in range(L):
        for s in range(1, t + 1):
            want[t] += (K[s - 1] @ Q[t]) * V[s]
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-11, atol=1e-11)


def test_per_channel_inner_product_closed_form(oracle_mod):
    """Falcon-2A, lambda=0, eps=0, unit keys: eta_{t,j} = beta_{t,j}, so
    o_{t,j} = sum_{s<=t} beta_{s,j} (x_s.q_t) v_{s,j}  ([NEWS] 02 (2): one rate
    per value channel)."""
    L, dk, dv = 25, 6, 4
    q, k, v, beta, _ = rnd(17, 1, 1, L, dk, dv, "F2A")
    out, _ = oracle_mod.fwd("F2A", "recurrent", q, k, v, beta, [0.0], 0.0)
    Q, V, Bt = q[0, 0], v[0, 0], beta[0, 0]
    X = np.zeros((L, dk))
    X[1:] = _phi(k[0, 0, :-1])
    want = np.tril(Q @ X.T) @ (Bt * V)
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("w", [2, 3, 5])
def test_window_inner_product_coefficients(oracle_mod, w):
    """Falcon-3A, lambda=0, eps=0, unit keys: eta_t = beta_t / |W_t'| (number of
    non-empty samples in the window, "block normalisation", [EXPL] 核心方法 2
    table) and o_t = sum_i c_{t,i} (x_i.q_t) y_i with
    c_{t,i} = sum_{s=i}^{min(t, i+w-1)} eta_s."""
    L, dk, dv = 20, 5, 3
    q, k, v, beta, _ = rnd(19, 1, 1, L, dk, dv, "F3A")
    out, _ = oracle_mod.fwd("F3A", "recurrent", q, k, v, beta, [0.0], 0.0, window=w)
    Q, V, Bt = q[0, 0], v[0, 0], beta[0, 0]
    X = np.zeros((L, dk))
    X[1:] = _phi(k[0, 0, :-1])
    nonempty = [sum(1 for i in range(max(0, s - w + 1), s + 1) if i >= 1) for s in range(L)]
    eta = [Bt[s] / nonempty[s] if nonempty[s] else 0.0 for s in range(L)]
    C = np.zeros((L, L))
    for t in range(L):
        for i in range(t + 1):
            C[t, i] = sum(eta[s] for s in range(i, min(t, i + w - 1) + 1))
    want = (C * (Q @ X.T)) @ V
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("variant", ["F1", "F2"])
def test_ridge_fixed_point_geometric(oracle_mod, variant):
    """Constant unit key x, constant target y, constant step: S_t = s_t x^T with
    s_t = s* (1 - rho^(t-1)), s* = y / (1 + lambda), rho = 1 - eta (1 + lambda),
    the L2-regularised regression of [NEWS] 02 (1) solved in closed form
    (per value channel for Falcon-2, [NEWS] 02 (2))."""
    L, dk, dv, lam, eps = 30, 6, 4, 0.3, 1e-3
    rng = np.random.default_rng(23)
    k = np.tile(rng.standard_normal(dk), (1, 1, L, 1))
    y = rng.standard_normal(dv)
    v = np.tile(y, (1, 1, L, 1))
    q = rng.standard_normal((1, 1, L, dk))
    bc = rng.uniform(0.2, 0.9, dv) if variant == "F2" else np.full(dv, 0.6)
    beta = np.tile(bc, (1, 1, L, 1)) if variant == "F2" else np.full((1, 1, L), 0.6)
    out, S = oracle_mod.fwd(variant, "recurrent", q, k, v, beta, [lam], eps)
    x = k[0, 0, 0] / np.linalg.norm(k[0, 0, 0])
    eta = bc / (eps + 1.0)
    rho = 1 - eta * (1 + lam)
    t = np.arange(1, L + 1)[:, None]
    s = (y / (1 + lam)) * (1 - rho[None, :] ** (t - 1))
    np.testing.assert_allclose(out[0, 0], s * (q[0, 0] @ x)[:, None], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], np.outer(s[-1], x), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("w", [2, 4])
def test_window_regression_constant_key(oracle_mod, w):
    """Falcon-3 with a constant unit key: the state stays s_t x^T and the window
    update collapses to s_t = alpha_t s_{t-1} + eta_t sum_{i in W_t, i>=2} (y_i - s_{t-1})
    with eta_t = beta_t / (eps + m_t), m_t the non-empty samples of W_t
    ("sliding-window mini-batch, block normalisation", [EXPL] 核心方法 2;
    [NEWS] 02 (2)).  Also: lambda=0, beta=1, eps=0 makes m_t eta_t = 1, i.e.
    s_t equals the window's mean target."""
    L, dk, dv, lam, eps = 18, 5, 3, 0.2, 1e-2
    rng = np.random.default_rng(29)
    k = np.tile(rng.standard_normal(dk), (1, 1, L, 1))
    v = rng.standard_normal((1, 1, L, dv))
    q = rng.standard_normal((1, 1, L, dk))
    beta = rng.uniform(0.1, 0.9, (1, 1, L))
    out, _ = oracle_mod.fwd("F3", "recurrent", q, k, v, beta, [lam], eps, window=w)
    x = k[0, 0, 0] / np.linalg.norm(k[0, 0, 0])
    s = np.zeros(dv)
    for t in range(L):  # 0-based; sample 0 is empty (x_1 = 0)
        Wn = [i for i in range(max(0, t - w + 1), t + 1) if i >= 1]
        if Wn:
            eta = beta[0, 0, t] / (eps + len(Wn))
            s = (1 - eta * lam) * s + eta * sum(v[0, 0, i] - s for i in Wn)
        np.testing.assert_allclose(out[0, 0, t], s * (q[0, 0, t] @ x), rtol=1e-10, atol=1e-12)
    out2, _ = oracle_mod.fwd("F3", "recurrent", q, k, v, np.ones((1, 1, L)), [0.0], 0.0, window=w)
    for t in range(1, L):
        Wn = [i for i in range(max(0, t - w + 1), t + 1) if i >= 1]
        mean = np.mean([v[0, 0, i] for i in Wn], axis=0)
        np.testing.assert_allclose(out2[0, 0, t], mean * (q[0, 0, t] @ x), rtol=1e-10, atol=1e-12)


def test_inner_product_constant_key(oracle_mod):
    """Inner-product family, constant key, lambda=0: S_t = (sum_s eta_s y_s) x^T
    ([NEWS] 02 (1): the A family writes the target directly, no erase)."""
    L, dk, dv = 15, 4, 3
    rng = np.random.default_rng(31)
    k = np.tile(rng.standard_normal(dk), (1, 1, L, 1))
    v = rng.standard_normal((1, 1, L, dv))
    q = rng.standard_normal((1, 1, L, dk))
    beta = rng.uniform(0.1, 0.9, (1, 1, L))
    _, S = oracle_mod.fwd("F1A", "recurrent", q, k, v, beta, [0.0], 1e-6)
    x = k[0, 0, 0] / np.linalg.norm(k[0, 0, 0])
    eta = beta[0, 0] / (1e-6 + 1.0)
    eta[0] = 0.0
    np.testing.assert_allclose(S[0, 0], np.outer((eta[:, None] * v[0, 0]).sum(0), x), rtol=1e-11)


def test_contraction_bound(oracle_mod):
    """Unit inputs and eta <= 1 make every regression transition
    alpha I - eta x x^T a contraction, so with bounded targets the state norm
    stays bounded by max|y| / min step ... checked as |S_t x| never exceeding
    max |y| / (1 - max alpha deficit) on a long random run (no blow-up; the
    positive decay of [EXPL] 核心方法 4 / [SUMM] 计算形式与数值稳定)."""
    L, dk, dv = 400, 8, 4
    q, k, v, beta, lam = rnd(37, 1, 1, L, dk, dv, "F1", lam_hi=0.05)
    _, S = oracle_mod.fwd("F1", "recurrent", q, k, v, beta, lam, 1e-6)
    # each row of S is a convex-like mixture of past targets along unit keys;
    # its spectral norm cannot exceed sum of |y| weighted by a geometric series
    assert np.linalg.norm(S[0, 0], 2) < np.abs(v).max() * np.sqrt(dv) * 50


# ---------------------------------------------------------------- variant reductions

def test_window_one_and_uniform_channels_reduce_to_falcon1(oracle_mod):
    """Falcon-3/3A with a window of one sample are Falcon-1/1A; Falcon-2/2A with
    the same gain on every channel are Falcon-1/1A ([EXPL] 核心方法 2 table:
    the variants differ only in granularity)."""
    L, dk, dv = 33, 8, 6
    q, k, v, beta, lam = rnd(41, 2, 2, L, dk, dv, "F1")
    for base, win_v, ch_v in (("F1", "F3", "F2"), ("F1A", "F3A", "F2A")):
        o1, S1 = oracle_mod.fwd(base, "recurrent", q, k, v, beta, lam, 1e-6)
        o3, S3 = oracle_mod.fwd(win_v, "recurrent", q, k, v, beta, lam, 1e-6, window=1)
        o2, S2 = oracle_mod.fwd(ch_v, "recurrent", q, k, v, np.repeat(beta[..., None], dv, -1), lam, 1e-6)
        for o, S in ((o3, S3), (o2, S2)):
            np.testing.assert_allclose(o, o1, rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(S, S1, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- decode

@pytest.mark.parametrize("pairing", ["prefix", "same_step"])
@pytest.mark.parametrize("variant", VARIANTS)
def test_decode_chain_equals_prefill(oracle_mod, variant, pairing):
    """prefill(L0) -> carry -> n decode steps == prefill(L0 + n): the fixed-size
    state plus the carry is the whole memory ([SUMM] 计算形式与数值稳定: the
    recurrent form for autoregressive inference), under either pairing (the
    same-step pair of [EXPL] 核心方法 1, warning paragraph, takes phi(k_t) as
    the step's own sample; the full run's samples come from the forward's
    pairing rule, written independently of the decode step)."""
    L0, n, dk, dv = 9, 7, 6, 4
    w = 3 if variant in ("F3", "F3A") else 1
    q, k, v, beta, lam = rnd(43, 2, 3, L0 + n, dk, dv, variant)
    o_full, S_full = oracle_mod.fwd(variant, "recurrent", q, k, v, beta, lam, 1e-6, window=w, pairing=pairing)
    _, S0 = oracle_mod.fwd(variant, "recurrent", q[:, :, :L0], k[:, :, :L0], v[:, :, :L0],
                           beta[:, :, :L0], lam, 1e-6, window=w, pairing=pairing)
    x_prev, win = oracle_mod.carry_from_prefill(variant, k[:, :, :L0], v[:, :, :L0], w, pairing=pairing)
    if pairing == "same_step":
        x_prev = None  # not read by the same-step step
    state = np.ascontiguousarray(S0)
    for t in range(L0, L0 + n):
        o = oracle_mod.decode_step(variant, q[:, :, t], k[:, :, t], v[:, :, t], beta[:, :, t],
                                   lam, 1e-6, w, state, x_prev, win, pairing=pairing)
        np.testing.assert_allclose(o, o_full[:, :, t], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(state, S_full, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("pairing", ["prefix", "same_step"])
@pytest.mark.parametrize("variant", VARIANTS)
def test_decode_from_zero_carry(oracle_mod, variant, pairing):
    """Decode from S=0 and an all-zero carry reproduces the sequence from its
    first token (prefix pair: x_1 = 0, the first step writes nothing; the
    same-step pair writes with phi(k_1) from the first step on)."""
    L, dk, dv = 8, 4, 3
    w = 3 if variant in ("F3", "F3A") else 1
    q, k, v, beta, lam = rnd(47, 1, 2, L, dk, dv, variant)
    o_full, S_full = oracle_mod.fwd(variant, "recurrent", q, k, v, beta, lam, 1e-6, window=w, pairing=pairing)
    state = np.zeros((1, 2, dv, dk))
    x_prev = np.zeros((1, 2, dk))
    win = np.zeros((1, 2, max(w - 1, 0), dk + dv))
    for t in range(L):
        o = oracle_mod.decode_step(variant, q[:, :, t], k[:, :, t], v[:, :, t], beta[:, :, t],
                                   lam, 1e-6, w, state, x_prev, win, pairing=pairing)
        np.testing.assert_allclose(o, o_full[:, :, t], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(state, S_full, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- edge cases

def test_edge_cases(oracle_mod):
    """L=0 (nothing), L=1 (x_1 = 0: output and state stay 0), zero keys
    (phi(0) = 0 writes nothing, eta = 0 by the reading for an empty sample)."""
    q, k, v, beta, lam = rnd(53, 1, 1, 1, 4, 3, "F1")
    o, S = oracle_mod.fwd("F1", "recurrent", q, k, v, beta, lam, 1e-6)
    assert np.all(o == 0) and np.all(S == 0)
    o, S = oracle_mod.fwd("F1", "chunk", q[:, :, :0], k[:, :, :0], v[:, :, :0], beta[:, :, :0], lam, 1e-6)
    assert o.shape == (1, 1, 0, 3) and np.all(S == 0)
    q, k, v, beta, lam = rnd(59, 1, 1, 6, 4, 3, "F1")
    k[:] = 0.0
    for var in VARIANTS:
        b = np.repeat(beta[..., None], 3, -1) if var in ("F2", "F2A") else beta
        o, S = oracle_mod.fwd(var, "recurrent", q, k, v, b, lam, 1e-6, window=wnd(var))
        assert np.all(o == 0) and np.all(S == 0)


# ---------------------------------------------------------------- segments continuing a sequence

def _carry_inputs(seed, B, H, dk, dv, variant):
    rng = np.random.default_rng(seed)
    S0 = rng.standard_normal((B, H, dv, dk)) * 0.5
    xp = rng.standard_normal((B, H, dk))
    xp /= np.linalg.norm(xp, axis=-1, keepdims=True)
    w = wnd(variant)
    win = rng.standard_normal((B, H, w - 1, dk + dv))
    win[..., :dk] /= np.linalg.norm(win[..., :dk], axis=-1, keepdims=True)
    return S0, xp, (win if w > 1 else None)


@pytest.mark.parametrize("variant", VARIANTS)
def test_carry_brute_force(oracle_mod, variant):
    """A segment entered with state S0 and the samples before it: the oracle's
    recurrence == the unrolled products S_t = S0 M_1...M_t + sum_s b_s
    M_{s+1}...M_t of the same per-step updates ([EXPL] 核心方法 1)."""
    L, dk, dv = 9, 4, 3
    q, k, v, beta, lam = rnd(21, 1, 2, L, dk, dv, variant, lam_hi=0.3)
    S0, xp, win = _carry_inputs(22, 1, 2, dk, dv, variant)
    w = wnd(variant)
    o, S = oracle_mod.fwd_carry(variant, q, k, v, beta, lam, 1e-6, window=w, S0=S0, x_prev=xp, win=win)
    assert np.abs(o).max() > 1e-2
    for h in range(2):
        bo, bS = brute.unit(variant, q[0, h], k[0, h], v[0, h], beta[0, h], float(lam[h]), 1e-6, w,
                            S0=S0[0, h], x_prev=xp[0, h], carry=None if win is None else win[0, h])
        np.testing.assert_allclose(o[0, h], bo, rtol=1e-9, atol=1e-10)
        np.testing.assert_allclose(S[0, h], bS, rtol=1e-9, atol=1e-10)


@pytest.mark.parametrize("variant", VARIANTS)
def test_carry_of_zeros_is_a_fresh_sequence(oracle_mod, variant):
    """Zero state and zero carry are the start of a sequence (x_1 = 0 and
    empty window samples add no energy and no gradient)."""
    q, k, v, beta, lam = rnd(23, 2, 2, 30, 8, 4, variant)
    w = wnd(variant)
    o0, S0_ = oracle_mod.fwd(variant, "recurrent", q, k, v, beta, lam, 1e-6, window=w)
    o1, S1 = oracle_mod.fwd_carry(variant, q, k, v, beta, lam, 1e-6, window=w)
    np.testing.assert_allclose(o1, o0, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S1, S0_, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("pairing", ["prefix", "same_step"])
@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("split", [1, 17, 40])
def test_continuation_equals_one_run(oracle_mod, variant, split, pairing):
    """Running a sequence in two segments -- the second one entered with the
    first one's final state and decode carry -- equals one run over the whole
    sequence (chunk form for the whole run, recurrent for the segments),
    under either pairing."""
    L, dk, dv = 57, 8, 4
    q, k, v, beta, lam = rnd(24, 2, 3, L, dk, dv, variant)
    w = 3 if variant in ("F3", "F3A") else 1
    o_all, S_all = oracle_mod.fwd(variant, "chunk", q, k, v, beta, lam, 1e-6, window=w, chunk=16, pairing=pairing)
    a = slice(0, split)
    b_ = slice(split, L)
    o1, S1 = oracle_mod.fwd(variant, "recurrent", q[:, :, a], k[:, :, a], v[:, :, a], beta[:, :, a], lam,
                            1e-6, window=w, pairing=pairing)
    xp, win = oracle_mod.carry_from_prefill(variant, k[:, :, a], v[:, :, a], w, pairing=pairing)
    if pairing == "same_step":
        xp = None  # the segment's first sample is its own phi(k)
    o2, S2 = oracle_mod.fwd_carry(variant, q[:, :, b_], k[:, :, b_], v[:, :, b_], beta[:, :, b_], lam, 1e-6,
                                  window=w, S0=S1, x_prev=xp, win=win, pairing=pairing)
    np.testing.assert_allclose(np.concatenate([o1, o2], 2), o_all, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(S2, S_all, rtol=1e-9, atol=1e-11)
