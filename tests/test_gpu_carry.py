"""GPU parity of falcon_fwd_carry: a segment that continues a sequence from an
initial state and the decode carry, against the fp64 oracle's recurrence
over the same carried samples (oracle.fwd_carry), and two segments against
one run over the whole sequence.

Error metric per tensor: max|gpu - oracle| / max|oracle|; bars 1e-4 (fp32
inputs) and 2e-2 (bf16 inputs), as for the other parity tests.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_sequence_falcon_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


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


def window_of(variant):
    return 3 if variant in ("F3", "F3A") else 1


def carry_inputs(seed, B, H, dk, dv, variant):
    """A state and carry as a real earlier segment would leave them: fp32,
    unit-norm samples, zeros nowhere."""
    rng = np.random.default_rng(seed)
    S0 = (rng.standard_normal((B, H, dv, dk)) * 0.5).astype(np.float32)
    xp = rng.standard_normal((B, H, dk))
    xp = (xp / np.linalg.norm(xp, axis=-1, keepdims=True)).astype(np.float32)
    w = window_of(variant)
    win = None
    if w > 1:
        win = rng.standard_normal((B, H, w - 1, dk + dv))
        win[..., :dk] /= np.linalg.norm(win[..., :dk], axis=-1, keepdims=True)
        win = win.astype(np.float32)
    return S0, xp, win


def check_segment(F, variant, form, dtype, B, H, L, dk, dv, chunk, seed, pairing="prefix"):
    """A segment entered with a state and carry.  Under the same-step pair
    the x_prev handed in is a random vector the segment must not read."""
    w = window_of(variant)
    d = gen.draw(variant, B, H, L, dk, dv, seed=seed, dtype=dtype)
    S0, xp, win = carry_inputs(seed + 1, B, H, dk, dv, variant)
    t = lambda a: None if a is None else torch.from_numpy(a).cuda()
    out, S = F.fwd(variant, form, *(d[n].cuda() for n in ("q", "k", "v", "beta", "lam")), d["eps"], window=w,
                   chunk=chunk, initial_state=t(S0), x_prev=t(xp), win=t(win), pairing=pairing)
    torch.cuda.synchronize()
    oo, oS = oracle.fwd_carry(variant, d["q_64"], d["k_64"], d["v_64"], d["beta_64"], d["lam_64"], d["eps_64"],
                              window=w, S0=S0.astype(np.float64),
                              x_prev=None if pairing == "same_step" else xp.astype(np.float64),
                              win=None if win is None else win.astype(np.float64), pairing=pairing)
    assert np.abs(oo).max() > 1e-3
    assert rel(out.double().cpu().numpy(), oo) <= TOL[dtype]
    assert rel(S.double().cpu().numpy(), oS) <= TOL[dtype]


# the tensor-core chunk paths: Falcon-1/1A, d = 64, chunk 16/32/64/128, bf16 (ragged tail, several chunks)
@pytest.mark.parametrize("chunk", [16, 32, 64, 128])
@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_carry_tensor_core_path(F, variant, chunk):
    check_segment(F, variant, "chunk", "bf16", 2, 3, 200, 64, 64, chunk, 31)


@pytest.mark.parametrize("d,chunk", [(32, 128), (128, 16), (128, 64)])
@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_carry_tensor_core_widths(F, variant, d, chunk):
    """A continued segment through the per-head chunk kernel at d = 32 and 128."""
    check_segment(F, variant, "chunk", "bf16", 1, 2, 200, d, d, chunk, 33)


@pytest.mark.parametrize("variant", ["F1", "F2", "F3", "F1A", "F2A", "F3A"])
@pytest.mark.parametrize("form,chunk", [("recurrent", 64), ("chunk", 32), ("chunk", 64)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_carry_span_and_recurrent(F, variant, form, chunk, dtype):
    check_segment(F, variant, form, dtype, 1, 2, 97, 32, 16, chunk, 41)


@pytest.mark.parametrize("pairing", ["prefix", "same_step"])
@pytest.mark.parametrize("variant", ["F1", "F2", "F3", "F1A", "F2A", "F3A"])
@pytest.mark.parametrize("form,dtype,dk", [("chunk", "bf16", 64), ("chunk", "f32", 32), ("recurrent", "bf16", 64)])
def test_two_segments_equal_one_run(F, variant, form, dtype, dk, pairing):
    """prefill(segment 1) -> final state + decode carry -> a continued
    segment 2 == the oracle over the whole sequence, under either pairing."""
    B, H, L, split = 2, 2, 230, 137
    dv = dk
    w = window_of(variant)
    d = gen.draw(variant, B, H, L, dk, dv, seed=51, dtype=dtype)
    a, b = slice(0, split), slice(split, L)
    seg = lambda sl: [d[n][:, :, sl].contiguous().cuda() for n in ("q", "k", "v", "beta")]
    lam = d["lam"].cuda()
    o1, S1 = F.fwd(variant, form, *seg(a), lam, d["eps"], window=w, chunk=64, pairing=pairing)
    q1, k1, v1, _ = seg(a)
    xp, win = F.carry_from_prefill(variant, k1, v1, w, pairing=pairing)
    o2, S2 = F.fwd(variant, form, *seg(b), lam, d["eps"], window=w, chunk=64, initial_state=S1, x_prev=xp, win=win,
                   pairing=pairing)
    torch.cuda.synchronize()
    oo, oS = oracle.fwd(variant, "recurrent", d["q_64"], d["k_64"], d["v_64"], d["beta_64"], d["lam_64"],
                        d["eps_64"], window=w, pairing=pairing)
    got = np.concatenate([o1.double().cpu().numpy(), o2.double().cpu().numpy()], 2)
    assert rel(got, oo) <= TOL[dtype]
    assert rel(S2.double().cpu().numpy(), oS) <= TOL[dtype]


def test_carry_rejected_for_the_masked_form(F):
    d = gen.draw("F1", 1, 1, 16, 32, 32, seed=5, dtype="f32")
    S0 = torch.zeros((1, 1, 32, 32), device="cuda")
    with pytest.raises(F.FalconError):
        F.fwd("F1", "masked", *(d[n].cuda() for n in ("q", "k", "v", "beta", "lam")), d["eps"], initial_state=S0)


def test_empty_segment_keeps_the_state(F):
    d = gen.draw("F2A", 1, 2, 0, 32, 16, seed=6, dtype="f32")
    S0 = torch.randn((1, 2, 16, 32), device="cuda")
    _, S = F.fwd("F2A", "chunk", *(d[n].cuda() for n in ("q", "k", "v", "beta", "lam")), d["eps"], initial_state=S0)
    torch.cuda.synchronize()
    assert torch.equal(S, S0)


def test_carry_falcon2a_d128_tensor_core_path(F):
    check_segment(F, "F2A", "chunk", "bf16", 1, 3, 200, 128, 128, 64, 81)


def test_carry_falcon2_d128_tensor_core_path(F):
    check_segment(F, "F2", "chunk", "bf16", 1, 3, 200, 128, 128, 64, 91)


@pytest.mark.parametrize("variant", ["F3", "F3A"])
def test_carry_window_tensor_core_path(F, variant):
    """window 3: the carried window samples (values included) and x_prev
    enter the first chunk's sample rows."""
    check_segment(F, variant, "chunk", "bf16", 1, 3, 200, 64, 64, 64, 141)


# ---- the same-step pair on every path that takes a carry
@pytest.mark.parametrize("variant,dk,dv", [("F1", 64, 64), ("F1A", 64, 64), ("F2A", 128, 128), ("F2", 128, 128),
                                           ("F3", 64, 64), ("F3A", 64, 64)])
def test_carry_same_step_tensor_core_paths(F, variant, dk, dv):
    check_segment(F, variant, "chunk", "bf16", 1, 3, 200, dk, dv, 64, 151, pairing="same_step")


@pytest.mark.parametrize("variant", ["F1", "F2", "F3", "F1A", "F2A", "F3A"])
@pytest.mark.parametrize("form,chunk", [("recurrent", 64), ("chunk", 32)])
def test_carry_same_step_span_and_recurrent(F, variant, form, chunk):
    check_segment(F, variant, form, "f32", 1, 2, 97, 32, 16, chunk, 161, pairing="same_step")
