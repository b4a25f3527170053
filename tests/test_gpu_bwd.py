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
