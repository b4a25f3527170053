"""falcon_fwd_host (inputs and outputs in host memory, the batch cut into
slices whose copies overlap the compute on two library-owned copy streams)
against falcon_fwd_ex on device buffers.  Each slice runs the same kernels on
its own batch rows, and every (b, h) is computed independently of the others,
so the two agree bit for bit."""
import pytest
import torch

from linear_attention_sequence_falcon_b200 import inputs as gen

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "beta", "lam")


@pytest.fixture(scope="module")
def F():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from linear_attention_sequence_falcon_b200 import build
    build.build()
    import linear_attention_sequence_falcon_b200 as F
    F.load()
    return F


def on_device(F, variant, form, d, **kw):
    out, st = F.fwd(variant, form, *(d[n].cuda() for n in NAMES), d["eps"], **kw)
    torch.cuda.synchronize()
    return out.cpu(), st.cpu()


def on_host(F, variants, form, d, pinned=True, **kw):
    h = [d[n].pin_memory() if pinned else d[n].clone() for n in NAMES]
    outs, states = F.fwd_host(variants, form, *h, d["eps"], **kw)
    torch.cuda.synchronize()
    return outs, states


@pytest.mark.parametrize("slices", [0, 1, 2, 3, 5])
def test_host_chunk_falcon1_pair(F, slices):
    """The tensor-core chunk path of Falcon-1 and Falcon-1A from one set of
    host inputs; B = 5 cut into 1..5 slices (uneven for 2 and 3)."""
    d = gen.draw("F1", 5, 3, 200, 64, 64, seed=300, dtype="bf16")
    outs, states = on_host(F, ["F1", "F1A"], "chunk", d, chunk=64, slices=slices)
    for i, var in enumerate(["F1", "F1A"]):
        ro, rs = on_device(F, var, "chunk", d, chunk=64)
        assert torch.equal(outs[i], ro), var
        assert torch.equal(states[i], rs), var


@pytest.mark.parametrize("slices", [0, 3])
def test_host_chunk_falcon3_pair_window(F, slices):
    """Falcon-3 and Falcon-3A (per-chunk images and the chain kernel, in the
    workspace the host call sizes) from one set of host inputs, window 4,
    B = 4 in 1 or 3 slices."""
    d = gen.draw("F3", 4, 3, 150, 64, 64, seed=302, dtype="bf16")
    outs, states = on_host(F, ["F3", "F3A"], "chunk", d, chunk=64, window=4, slices=slices)
    for i, var in enumerate(["F3", "F3A"]):
        ro, rs = on_device(F, var, "chunk", d, chunk=64, window=4)
        assert torch.equal(outs[i], ro), var
        assert torch.equal(states[i], rs), var


def test_host_per_channel_pair_pageable(F):
    """Falcon-2 and Falcon-2A (per-channel beta), recurrent fp32, from
    pageable host memory."""
    d = gen.draw("F2", 3, 2, 50, 32, 32, seed=301, dtype="f32")
    outs, states = on_host(F, ["F2", "F2A"], "recurrent", d, pinned=False, slices=2)
    for i, var in enumerate(["F2", "F2A"]):
        ro, rs = on_device(F, var, "recurrent", d)
        assert torch.equal(outs[i], ro), var
        assert torch.equal(states[i], rs), var


def test_host_window_chunk_and_pairing(F):
    """Falcon-3 with a window of 3 (chunk path), and the same-step pairing
    with the identity map for Falcon-3A."""
    d = gen.draw("F3", 2, 3, 130, 64, 64, seed=302, dtype="bf16")
    outs, states = on_host(F, ["F3"], "chunk", d, chunk=64, window=3, slices=2)
    ro, rs = on_device(F, "F3", "chunk", d, chunk=64, window=3)
    assert torch.equal(outs[0], ro) and torch.equal(states[0], rs)
    outs, states = on_host(F, ["F3A"], "masked", d, window=2, slices=2, pairing="same_step", phi="identity")
    ro, rs = on_device(F, "F3A", "masked", d, window=2, pairing="same_step", phi="identity")
    assert torch.equal(outs[0], ro) and torch.equal(states[0], rs)


def test_host_workload2_shape(F):
    """The 8x12x2048x64 bf16 shape with the library's slice count."""
    d = gen.draw("F1", 8, 12, 2048, 64, 64, seed=303, dtype="bf16")
    outs, states = on_host(F, ["F1", "F1A"], "chunk", d, chunk=64)
    for i, var in enumerate(["F1", "F1A"]):
        ro, rs = on_device(F, var, "chunk", d, chunk=64)
        assert torch.equal(outs[i], ro), var
        assert torch.equal(states[i], rs), var


def test_host_empty_sequence_and_no_state(F):
    d = gen.draw("F1A", 2, 3, 0, 64, 64, seed=304, dtype="bf16")
    outs, states = on_host(F, ["F1A"], "chunk", d, chunk=64)
    assert outs[0].shape == (2, 3, 0, 64)
    assert torch.count_nonzero(states[0]) == 0
    d = gen.draw("F1A", 2, 3, 40, 64, 64, seed=305, dtype="bf16")
    outs, states = on_host(F, ["F1A"], "recurrent", d, want_state=False)
    assert states is None
    ro, _ = on_device(F, "F1A", "recurrent", d)
    assert torch.equal(outs[0], ro)


def test_host_rejects_mixed_beta_layouts(F):
    d = gen.draw("F1", 1, 1, 8, 32, 32, seed=306, dtype="f32")
    with pytest.raises(F.FalconError):
        on_host(F, ["F1", "F2"], "recurrent", d)
