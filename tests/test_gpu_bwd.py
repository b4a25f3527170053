"""GPU parity of falcon_bwd (the backward pass of every variant)
against the fp64 oracle's reverse mode of the recurrent definition
(oracle.bwd, pinned by finite differences in test_oracle_bwd.py), on the same
seeded inputs.

Error metric per gradient: max|gpu - oracle| / max|oracle|.  The GPU path
computes in fp32 from the (bf16-rounded) inputs the oracle also receives, so
one bar serves both dtypes: 1e-4, over sums of up to a few thousand terms.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_sequence_falcon_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL = 1e-4
NAMES = ("dq", "dk", "dv", "dbeta", "dlambda")


@pytest.fixture(scope="module")
def F():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from linear_attention_sequence_falcon_b200 import build
    build.build()
    import linear_attention_sequence_falcon_b200 as F
    F.load()
    return F


def rel(gpu, ref):
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(np.asarray(gpu, dtype=np.float64) - ref).max() / max(np.abs(ref).max(), 1e-30))


def grads_case(F, variant, B, H, L, d, dtype, seed, pairing="prefix", phi="l2", with_dstate=True, lam=None,
               key_scale=1.0, units=None, window=None):
    if window is None:
        window = 3 if variant in ("F3", "F3A") else 1
    d_ = gen.draw(variant, B, H, L, d, d, seed=seed, dtype=dtype, lam=lam, key_scale=key_scale)
    rng = np.random.default_rng(seed + 1)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    do = torch.from_numpy(rng.standard_normal((B, H, L, d)).astype(np.float32)).to(tdt)
    ds = torch.from_numpy(rng.standard_normal((B, H, d, d)).astype(np.float32)) if with_dstate else None
    g = F.bwd(variant, *(d_[n].cuda() for n in ("q", "k", "v", "beta", "lam")), d_["eps"], do.cuda(),
              None if ds is None else ds.cuda(), window=window, pairing=pairing, phi=phi)
    torch.cuda.synchronize()
    if units is None:
        args = [d_[n] for n in ("q_64", "k_64", "v_64", "beta_64")]
        ref = oracle.bwd(variant, *args, d_["lam_64"], d_["eps_64"], do.double().numpy(),
                         None if ds is None else ds.double().numpy(), window=window, pairing=pairing, phi=phi)
        got = {n: g[n].double().cpu().numpy() for n in NAMES}
        return got, ref
    # sampled (b, h) units of a large case: each through the oracle as a batch of one
    got = {n: [] for n in NAMES if n != "dlambda"}
    ref = {n: [] for n in NAMES if n != "dlambda"}
    for b, h in units:
        one = lambda a: np.ascontiguousarray(a[b:b + 1, h:h + 1])  # noqa: E731
        r = oracle.bwd(variant, *(one(d_[n]) for n in ("q_64", "k_64", "v_64", "beta_64")),
                       np.asarray(d_["lam_64"])[h:h + 1], d_["eps_64"], one(do.double().numpy()),
                       None if ds is None else one(ds.double().numpy()), window=window, pairing=pairing, phi=phi)
        for n in got:
            got[n].append(g[n][b, h].double().cpu().numpy())
            ref[n].append(r[n][0, 0])
    return ({n: np.stack(v) for n, v in got.items()}, {n: np.stack(v) for n, v in ref.items()})


def check(got, ref, tol=TOL):
    for n in got:
        assert np.isfinite(got[n]).all(), n
        e = rel(got[n], ref[n])
        assert e <= tol, f"{n}: {e:.3e} (tol {tol})"


@pytest.mark.parametrize("variant", ["F1", "F2", "F3", "F1A", "F2A", "F3A"])
@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", [1, 37, 100])
def test_backward_parity(F, variant, d, dtype, L):
    """B=2, H=3: one token, a tile and a tail, three tiles and a tail."""
    got, ref = grads_case(F, variant, 2, 3, L, d, dtype, seed=200 + L + d)
    check(got, ref)


@pytest.mark.parametrize("variant", ["F1", "F2", "F3", "F1A", "F2A", "F3A"])
@pytest.mark.parametrize("pairing,phi", [("same_step", "l2"), ("prefix", "identity"), ("same_step", "identity")])
def test_backward_pairing_and_feature_map(F, variant, pairing, phi):
    got, ref = grads_case(F, variant, 1, 2, 70, 64, "f32", seed=231, pairing=pairing, phi=phi, key_scale=0.3)
    check(got, ref)


@pytest.mark.parametrize("variant", ["F1", "F2", "F3", "F1A", "F2A", "F3A"])
def test_backward_without_state_gradient_and_with_clamped_decay(F, variant):
    """dstate = NULL, and lambda = 0.9 with tiny keys under the identity map:
    eta = beta/(eps+|x|^2) is large, alpha sits on its 2^-20 floor for most
    tokens (no gradient through the clamp) and just above it for some.  There
    dalpha = (sum of dL/dG)/alpha divides an fp32 running sum by alpha down to
    2^-20, and the fp32 and fp64 sides may put a token on different sides of
    the floor, so this case takes 1e-3 instead of 1e-4."""
    got, ref = grads_case(F, variant, 1, 2, 90, 32, "f32", seed=241, with_dstate=False, lam=0.9,
                          phi="identity", key_scale=0.05)
    check(got, ref, tol=1e-3)


def test_backward_empty_sequence(F):
    d_ = gen.draw("F1A", 1, 2, 0, 64, 64, seed=1, dtype="f32")
    g = F.bwd("F1A", *(d_[n].cuda() for n in ("q", "k", "v", "beta", "lam")), d_["eps"],
              torch.zeros((1, 2, 0, 64), device="cuda"))
    torch.cuda.synchronize()
    assert torch.count_nonzero(g["dlambda"]) == 0


@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_backward_workload2_sampled(F, variant):
    """The workload-2 shape (8x12x2048x64 bf16): three sampled (b, h) units."""
    got, ref = grads_case(F, variant, 8, 12, 2048, 64, "bf16", seed=20260002, units=[(0, 0), (3, 7), (7, 11)])
    check(got, ref)


@pytest.mark.parametrize("w", [1, 2, 4, 8])
@pytest.mark.parametrize("variant", ["F3", "F3A"])
def test_backward_windows(F, variant, w):
    """Windows of 1, 2, 4 and 8 samples (the staged tile carries the 7 samples
    before it; each sample's gradient gathers the w steps that use it; a
    window of 1 runs the single-sample sweeps)."""
    got, ref = grads_case(F, variant, 1, 2, 75, 64, "f32", seed=250 + w, window=w)
    check(got, ref)


def test_backward_rejects_an_unsupported_shape(F):
    d_ = gen.draw("F1", 1, 1, 8, 64, 32, seed=2, dtype="f32")
    with pytest.raises(F.FalconError):
        F.bwd("F1", *(d_[n].cuda() for n in ("q", "k", "v", "beta", "lam")), d_["eps"],
              torch.zeros((1, 1, 8, 32), device="cuda"))


# --------------------------------------------------------------- the chunk-parallel backward (Falcon-1/1A, bf16, d = 64)

def _check_chunk(F, variant, B, H, L, seed, with_state=True, pairing="prefix", phi="l2", lam=None, key_scale=1.0,
                 units=None, tol=2e-2):
    kw = dict(dtype="bf16", key_scale=key_scale)
    if lam is not None:
        kw["lam"] = lam
    d = gen.draw(variant, B, H, L, 64, 64, seed=seed, **kw)
    rng = np.random.default_rng(seed + 1)
    do = torch.from_numpy(rng.standard_normal((B, H, L, 64)).astype(np.float32)).to(torch.bfloat16)
    ds = torch.from_numpy(rng.standard_normal((B, H, 64, 64)).astype(np.float32)) if with_state else None
    a = [d[k].cuda() for k in ("q", "k", "v", "beta", "lam")]
    g = F.bwd(variant, *a, d["eps"], do.cuda(), ds.cuda() if ds is not None else None, pairing=pairing, phi=phi,
              form="chunk", chunk=64)
    torch.cuda.synchronize()
    sel = (lambda x: x) if units is None else (lambda x: np.stack([x[b, h] for b, h in units]))
    if units is None:
        ref = oracle.bwd(variant, d["q_64"], d["k_64"], d["v_64"], d["beta_64"], d["lam_64"], d["eps_64"],
                         do.double().numpy(), None if ds is None else ds.double().numpy(), pairing=pairing, phi=phi)
    else:
        parts = []
        for (b, h) in units:
            s_ = lambda x: x[b:b + 1, h:h + 1]  # noqa: E731
            parts.append(oracle.bwd(variant, s_(d["q_64"]), s_(d["k_64"]), s_(d["v_64"]), s_(d["beta_64"]),
                                    d["lam_64"][h:h + 1], d["eps_64"], s_(do.double().numpy()),
                                    None if ds is None else s_(ds.double().numpy()), pairing=pairing, phi=phi))
        ref = {n: np.stack([p_[n][0, 0] for p_ in parts]) for n in ("dq", "dk", "dv", "dbeta")}
    for n in ("dq", "dk", "dv", "dbeta"):
        got = sel(g[n].double().cpu().numpy())
        e = rel(got, ref[n])
        assert np.isfinite(got).all() and e <= tol, (variant, n, e)
    if units is None:
        # dlambda is a sum over every token of -eta_t dL/dalpha_t; a sum whose
        # terms carry a relative error e is accurate to e times the mass of
        # its terms, which the oracle reports per head (terms of both signs
        # cancel under strong forgetting, so the sum itself can be far smaller)
        dl = g["dlambda"].double().cpu().numpy()
        assert np.all(np.abs(dl - ref["dlambda"]) <= tol * ref["dlambda_l1"]), (variant, dl, ref["dlambda"],
                                                                              ref["dlambda_l1"])


@pytest.mark.parametrize("variant", ["F1", "F1A"])
@pytest.mark.parametrize("L", [1, 64, 100, 257])
def test_chunk_backward_matches_oracle(F, variant, L):
    """One chunk, a ragged tail, several chunks: every gradient of the
    chunk-parallel backward against the reverse mode of the fp64 recurrence."""
    _check_chunk(F, variant, 2, 3, L, seed=900 + L)


@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_chunk_backward_without_state_gradient(F, variant):
    _check_chunk(F, variant, 1, 2, 200, seed=911, with_state=False)


@pytest.mark.parametrize("pairing,phi", [("same_step", "l2"), ("prefix", "identity")])
@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_chunk_backward_pairing_and_feature_map(F, variant, pairing, phi):
    _check_chunk(F, variant, 1, 2, 150, seed=913, pairing=pairing, phi=phi, key_scale=0.125)


@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_chunk_backward_strong_forgetting(F, variant):
    """lambda = 0.999: chunk log-decays around -45."""
    _check_chunk(F, variant, 1, 3, 200, seed=915, lam=0.999)


@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_chunk_backward_workload2_shape(F, variant):
    """8 x 12 x 2048 x 64 bf16, 32 chunks per head; three sampled heads
    against the oracle's reverse mode."""
    _check_chunk(F, variant, 8, 12, 2048, seed=917, units=[(0, 0), (3, 7), (7, 11)])


def test_chunk_backward_matches_recurrent_backward(F):
    """The two forms' gradients on the GPU agree (same function, two
    computations)."""
    d = gen.draw("F1", 2, 2, 300, 64, 64, seed=919, dtype="bf16")
    a = [d[k].cuda() for k in ("q", "k", "v", "beta", "lam")]
    do = torch.randn((2, 2, 300, 64), device="cuda").to(torch.bfloat16)
    ds = torch.randn((2, 2, 64, 64), device="cuda")
    g1 = F.bwd("F1", *a, d["eps"], do, ds, form="chunk")
    g2 = F.bwd("F1", *a, d["eps"], do, ds, form="recurrent")
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "dbeta"):
        assert rel(g1[n].double().cpu().numpy(), g2[n].double().cpu().numpy()) <= 2e-2, n
    # dlambda sums terms of both signs over every token: the two forms may
    # differ by the per-term error times the mass of the terms, which the
    # oracle reports for these inputs
    ref = oracle.bwd("F1", d["q_64"], d["k_64"], d["v_64"], d["beta_64"], d["lam_64"], d["eps_64"],
                     do.double().cpu().numpy(), ds.double().cpu().numpy())
    dl1, dl2 = (g["dlambda"].double().cpu().numpy() for g in (g1, g2))
    assert np.all(np.abs(dl1 - dl2) <= 2e-2 * ref["dlambda_l1"]), (dl1, dl2, ref["dlambda_l1"])
