"""GPU parity: the CUDA path, called through the C ABI, against the fp64 oracle
on the same seeded inputs.

Error metric per tensor: max|gpu - oracle| / max|oracle| (max-norm relative).
Bars: 1e-4 for fp32 inputs, 2e-2 for bf16 inputs with fp32 accumulation and
state.  The oracle reference for every form is the recurrent definition.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_sequence_falcon_b200 import inputs as gen

pytestmark = pytest.mark.gpu

VARIANTS = ("F1", "F2", "F3", "F1A", "F2A", "F3A")
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
    den = max(np.abs(ref).max(), 1e-30)
    return float(np.abs(np.asarray(gpu, dtype=np.float64) - ref).max() / den)


def dev(d, name):
    return d[name].cuda()


def gpu_fwd(F, d, variant, form, chunk=64, window=1, pairing="prefix", phi="l2"):
    out, S = F.fwd(variant, form, dev(d, "q"), dev(d, "k"), dev(d, "v"), dev(d, "beta"), dev(d, "lam"),
                   d["eps"], window=window, chunk=chunk, pairing=pairing, phi=phi)
    torch.cuda.synchronize()
    return out.double().cpu().numpy(), S.double().cpu().numpy()


def oracle_fwd(d, variant, window=1, units=None, pairing="prefix", phi="l2", form="recurrent", chunk=64):
    q, k, v, b = d["q_64"], d["k_64"], d["v_64"], d["beta_64"]
    lam = d["lam_64"]
    if units is None:
        return oracle.fwd(variant, form, q, k, v, b, lam, d["eps_64"], window=window, chunk=chunk,
                          pairing=pairing, phi=phi)
    outs, Ss = [], []
    for (bb, hh) in units:
        o, S = oracle.fwd(variant, form, q[bb:bb + 1, hh:hh + 1], k[bb:bb + 1, hh:hh + 1],
                          v[bb:bb + 1, hh:hh + 1], b[bb:bb + 1, hh:hh + 1], lam[hh:hh + 1], d["eps_64"],
                          window=window, chunk=chunk, pairing=pairing, phi=phi)
        outs.append(o[0, 0])
        Ss.append(S[0, 0])
    return np.stack(outs), np.stack(Ss)


def check(F, d, variant, form, chunk=64, window=1, units=None, pairing="prefix", phi="l2", tol=None):
    go, gS = gpu_fwd(F, d, variant, form, chunk, window, pairing, phi)
    oo, oS = oracle_fwd(d, variant, window, units, pairing, phi)
    if units is not None:
        go = np.stack([go[b, h] for b, h in units])
        gS = np.stack([gS[b, h] for b, h in units])
    tol = tol if tol is not None else TOL[d["dtype"]]
    eo, eS = rel(go, oo), rel(gS, oS)
    assert np.isfinite(go).all() and np.isfinite(gS).all()
    assert eo <= tol and eS <= tol, f"{variant} {form} C={chunk}: out {eo:.3e} state {eS:.3e} (tol {tol})"
    return eo, eS


# --------------------------------------------------------------- small shapes, every combination

@pytest.mark.parametrize("dk,dv", [(16, 16), (64, 64), (128, 128), (32, 64)])
@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("form", ["recurrent", "masked", "chunk"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_parity_small(F, dtype, form, variant, dk, dv):
    """B=2, H=3, L=150: several 64-token tiles and a ragged tail of 22."""
    d = gen.draw(variant, 2, 3, 150, dk, dv, seed=1000 + dk + dv, dtype=dtype)
    w = 4 if variant in ("F3", "F3A") else 1
    check(F, d, variant, form, chunk=64, window=w)


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("variant", VARIANTS)
def test_chunk_sizes(F, variant, chunk):
    """Chunk-size invariance: every chunk length against the recurrent oracle."""
    d = gen.draw(variant, 2, 2, 200, 64, 64, seed=77, dtype="bf16")
    w = 3 if variant in ("F3", "F3A") else 1
    check(F, d, variant, "chunk", chunk=chunk, window=w)


@pytest.mark.parametrize("chunk", [16, 32, 128])
@pytest.mark.parametrize("L", [1, 15, 100, 128, 129, 513])
@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_tensor_core_chunk_lengths(F, variant, L, chunk):
    """bf16 Falcon-1/1A at d = 64 with chunk 16, 32 and 128 (the tensor-core
    path that walks a head's chunks): one token, ragged tails, exact
    multiples and many chunks."""
    d = gen.draw(variant, 2, 3, L, 64, 64, seed=300 + L + chunk, dtype="bf16")
    check(F, d, variant, "chunk", chunk=chunk)


@pytest.mark.parametrize("chunk", [16, 32, 128])
@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_tensor_core_chunk_lengths_options(F, variant, chunk):
    """The same path with the same-step pair, the identity map, strong
    forgetting and the decay floor."""
    d = gen.draw(variant, 1, 2, 150, 64, 64, seed=310 + chunk, dtype="bf16", key_scale=0.125)
    check(F, d, variant, "chunk", chunk=chunk, pairing="same_step", phi="identity")
    d = gen.draw(variant, 1, 3, 200, 64, 64, seed=311 + chunk, dtype="bf16", lam=0.999)
    check(F, d, variant, "chunk", chunk=chunk)
    d = gen.draw(variant, 1, 2, 200, 64, 64, seed=312 + chunk, dtype="bf16", lam=0.9, key_scale=0.05)
    check(F, d, variant, "chunk", chunk=chunk, phi="identity")


@pytest.mark.parametrize("d_,chunk", [(32, 16), (32, 32), (32, 64), (32, 128), (128, 16), (128, 32), (128, 64)])
@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_tensor_core_chunk_widths(F, variant, d_, chunk):
    """The per-head tensor-core chunk kernel at d = 32 and d = 128: one token,
    a ragged tail and many chunks, with the same-step pair and strong
    forgetting on the longest case."""
    for L in (1, 100, 300):
        d = gen.draw(variant, 2, 2, L, d_, d_, seed=320 + L + chunk + d_, dtype="bf16")
        check(F, d, variant, "chunk", chunk=chunk)
    d = gen.draw(variant, 1, 2, 300, d_, d_, seed=330 + chunk + d_, dtype="bf16", lam=0.999, key_scale=0.125)
    check(F, d, variant, "chunk", chunk=chunk, pairing="same_step")


@pytest.mark.parametrize("w", [1, 2, 5, 8])
@pytest.mark.parametrize("variant", ["F3", "F3A"])
@pytest.mark.parametrize("form", ["recurrent", "masked", "chunk"])
def test_windows(F, variant, form, w):
    d = gen.draw(variant, 1, 2, 130, 32, 32, seed=90 + w, dtype="f32")
    check(F, d, variant, form, chunk=32, window=w)


@pytest.mark.parametrize("pairing,phi", [("same_step", "l2"), ("prefix", "identity"), ("same_step", "identity")])
@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("form", ["recurrent", "masked", "chunk"])
def test_pairing_and_feature_map(F, variant, form, pairing, phi):
    """The same-step pair and the identity feature map through falcon_fwd_ex."""
    d = gen.draw(variant, 1, 2, 100, 16, 16, seed=5, dtype="f32", key_scale=0.25)
    w = 3 if variant in ("F3", "F3A") else 1
    check(F, d, variant, form, chunk=32, window=w, pairing=pairing, phi=phi)


@pytest.mark.parametrize("L", [1, 2, 5, 63, 64, 65])
@pytest.mark.parametrize("form", ["recurrent", "masked", "chunk"])
def test_short_sequences(F, form, L):
    for variant in VARIANTS:
        d = gen.draw(variant, 1, 2, L, 64, 64, seed=L, dtype="f32")
        w = 3 if variant in ("F3", "F3A") else 1
        go, gS = gpu_fwd(F, d, variant, form, 64, w)
        oo, oS = oracle_fwd(d, variant, w)
        if L == 1:  # x_1 = 0: nothing is written
            assert np.abs(go).max() == 0 and np.abs(gS).max() == 0
        else:
            assert rel(go, oo) <= 1e-4 and rel(gS, oS) <= 1e-4


@pytest.mark.parametrize("form", ["recurrent", "masked", "chunk"])
def test_empty_sequence_zeroes_state(F, form):
    q = torch.zeros((2, 2, 0, 64), device="cuda", dtype=torch.bfloat16)
    v = torch.zeros((2, 2, 0, 64), device="cuda", dtype=torch.bfloat16)
    b = torch.zeros((2, 2, 0), device="cuda", dtype=torch.bfloat16)
    lam = torch.zeros(2, device="cuda")
    S = torch.full((2, 2, 64, 64), 7.0, device="cuda")
    F.fwd("F1", form, q, q, v, b, lam, 1e-6, final_state=S)
    torch.cuda.synchronize()
    assert float(S.abs().max()) == 0.0


@pytest.mark.parametrize("form", ["recurrent", "masked", "chunk"])
def test_zero_keys_write_nothing(F, form):
    for variant in VARIANTS:
        d = gen.draw(variant, 1, 2, 70, 32, 32, seed=3, dtype="bf16")
        d["k"] = torch.zeros_like(d["k"])
        go, gS = gpu_fwd(F, d, variant, form, 32, 3 if variant in ("F3", "F3A") else 1)
        assert np.abs(go).max() == 0 and np.abs(gS).max() == 0


def test_strong_forgetting_floor(F):
    """lambda close to 1 with tiny keys under the identity map drives
    1 - eta*lambda below zero; the positive-decay floor takes over."""
    for variant in VARIANTS:
        d = gen.draw(variant, 1, 2, 90, 16, 16, seed=8, dtype="f32", lam=0.9, key_scale=0.05)
        w = 2 if variant in ("F3", "F3A") else 1
        for form in ("recurrent", "masked", "chunk"):
            check(F, d, variant, form, chunk=16, window=w, phi="identity")


# --------------------------------------------------------------- the five benchmark workloads

def test_workload1_falcon1_recurrent_fp32(F):
    d = gen.workload_inputs(1, "F1")
    check(F, d, "F1", "recurrent", tol=1e-4)


@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_workload2_chunk_full(F, variant):
    """8x12x2048x64 bf16, chunk 64, every (b,h) unit against the oracle."""
    d = gen.workload_inputs(2, variant)
    check(F, d, variant, "chunk", chunk=64)


@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_workload2_masked_tensor_core(F, variant):
    """8x12x2048x64 bf16 in the masked-parallel form (the tensor-core pair
    products): sampled units against the oracle, and every unit against the
    chunk-parallel form on the GPU (the same function computed two ways)."""
    d = gen.workload_inputs(2, variant)
    check(F, d, variant, "masked", units=[(0, 0), (3, 7), (7, 11)])
    om, Sm = gpu_fwd(F, d, variant, "masked")
    oc, Sc = gpu_fwd(F, d, variant, "chunk")
    assert rel(om, oc) <= 2e-2 and rel(Sm, Sc) <= 2e-2


@pytest.mark.parametrize("L", [1, 63, 64, 65, 200, 700])
@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_masked_tensor_core_lengths(F, variant, L):
    """The masked-parallel tensor-core kernel (bf16, d = 64): one block, a
    ragged block, exact multiples and many row blocks."""
    d = gen.draw(variant, 2, 2, L, 64, 64, seed=340 + L, dtype="bf16")
    check(F, d, variant, "masked")


@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_masked_tensor_core_options(F, variant):
    """The same kernel with the same-step pair and the identity map, strong
    forgetting, and the decay floor."""
    d = gen.draw(variant, 1, 2, 300, 64, 64, seed=350, dtype="bf16", key_scale=0.125)
    check(F, d, variant, "masked", pairing="same_step", phi="identity")
    d = gen.draw(variant, 1, 3, 400, 64, 64, seed=351, dtype="bf16", lam=0.999)
    check(F, d, variant, "masked")
    d = gen.draw(variant, 1, 2, 300, 64, 64, seed=352, dtype="bf16", lam=0.9, key_scale=0.05)
    check(F, d, variant, "masked", phi="identity")


@pytest.mark.parametrize("L", [1, 60, 61, 62, 122, 123, 300])
@pytest.mark.parametrize("w", [2, 3, 4])
@pytest.mark.parametrize("variant", ["F3", "F3A"])
def test_masked_tensor_core_windows(F, variant, w, L):
    """The masked tensor-core kernel with windows (bf16, d = 64): row blocks
    of 65 - B_w tokens whose window samples fill 64 rows; one token, block
    edges and many blocks."""
    d = gen.draw(variant, 2, 2, L, 64, 64, seed=360 + L + 7 * w, dtype="bf16")
    check(F, d, variant, "masked", window=w)


@pytest.mark.parametrize("variant", ["F3", "F3A"])
def test_masked_tensor_core_window_options(F, variant):
    """Windowed masked form with the same-step pair and the identity map,
    strong forgetting, and the decay floor."""
    d = gen.draw(variant, 1, 2, 250, 64, 64, seed=370, dtype="bf16", key_scale=0.125)
    check(F, d, variant, "masked", window=3, pairing="same_step", phi="identity")
    d = gen.draw(variant, 1, 3, 300, 64, 64, seed=371, dtype="bf16", lam=0.999)
    check(F, d, variant, "masked", window=4)
    d = gen.draw(variant, 1, 2, 200, 64, 64, seed=372, dtype="bf16", lam=0.9, key_scale=0.05)
    check(F, d, variant, "masked", window=2, phi="identity")


@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_masked_misaligned_inputs_take_the_cuda_core_kernel(F, variant):
    """Inputs that are not 16-byte aligned (a view one element into its
    storage) are refused by the tensor-core kernel and computed by the
    CUDA-core one: same results within the tolerance."""
    d = gen.draw(variant, 1, 2, 130, 64, 64, seed=353, dtype="bf16")
    a = []
    for n in ("q", "k", "v", "beta", "lam"):
        x = dev(d, n)
        if n != "lam":
            buf = torch.empty(x.numel() + 1, dtype=x.dtype, device=x.device)
            buf[1:].copy_(x.reshape(-1))
            x = buf[1:].view(x.shape)
        a.append(x)
    out, S = F.fwd(variant, "masked", *a, d["eps"])
    torch.cuda.synchronize()
    oo, oS = oracle_fwd(d, variant)
    assert rel(out.double().cpu().numpy(), oo) <= TOL["bf16"] and rel(S.double().cpu().numpy(), oS) <= TOL["bf16"]


def test_workload3_falcon2_chunk_sampled(F):
    """4x16x4096x128 bf16, per-channel beta; sampled units."""
    d = gen.workload_inputs(3, "F2")
    check(F, d, "F2", "chunk", chunk=64, units=[(0, 0), (1, 7), (3, 15)])


@pytest.mark.parametrize("variant", ["F3", "F3A"])
@pytest.mark.parametrize("form", ["masked", "chunk"])
def test_workload4_window_full(F, variant, form):
    d = gen.workload_inputs(4, variant)
    check(F, d, variant, form, chunk=64, window=4, units=[(0, 0), (2, 5), (7, 11)])


def test_workload4_masked_equals_chunk(F):
    """The two parallel forms against each other on the full workload."""
    for variant in ("F3", "F3A"):
        d = gen.workload_inputs(4, variant)
        om, Sm = gpu_fwd(F, d, variant, "masked", 64, 4)
        oc, Sc = gpu_fwd(F, d, variant, "chunk", 64, 4)
        assert rel(om, oc) <= 2e-2 and rel(Sm, Sc) <= 2e-2


def test_workload5_prefill_sampled(F):
    """2x16x32768x128 bf16 Falcon-2A prefill; sampled units."""
    d = gen.workload_inputs(5, "F2A")
    check(F, d, "F2A", "chunk", chunk=64, units=[(0, 0), (1, 15)])


# --------------------------------------------------------------- decode

def _decode_chain(F, variant, N, H, dk, dv, L0, steps, dtype, w, pairing="prefix", lam=0.02, seed=555):
    d = gen.draw(variant, N, H, L0 + steps, dk, dv, seed=seed, dtype=dtype, lam=lam)
    pre = {n: d[n][:, :, :L0].contiguous() for n in ("q", "k", "v", "beta")}
    _, S = F.fwd(variant, "chunk", *(pre[n].cuda() for n in ("q", "k", "v", "beta")), d["lam"].cuda(), d["eps"],
                 window=w, chunk=64, pairing=pairing)
    x_prev, win = F.carry_from_prefill(variant, pre["k"].cuda(), pre["v"].cuda(), w, pairing=pairing)
    torch.cuda.synchronize()
    # carry parity
    ox, ow = oracle.carry_from_prefill(variant, d["k_64"][:, :, :L0], d["v_64"][:, :, :L0], w, pairing=pairing)
    assert rel(x_prev.double().cpu().numpy(), ox) <= 1e-6
    if w > 1:
        assert rel(win.double().cpu().numpy(), ow) <= 1e-6
    # every step's token vectors as one contiguous [steps, N, H, ...] block on the device
    tok = {n: d[n][:, :, L0:].movedim(2, 0).contiguous().cuda() for n in ("q", "k", "v", "beta")}
    lam_d = d["lam"].cuda()
    outs = torch.empty((steps,) + (N, H, dv), dtype=d["q"].dtype, device="cuda")
    for i in range(steps):
        F.decode_step(variant, tok["q"][i], tok["k"][i], tok["v"][i], tok["beta"][i], lam_d, d["eps"], w, S,
                      None if pairing == "same_step" else x_prev, win, out=outs[i], pairing=pairing)
    torch.cuda.synchronize()
    return d, outs.movedim(0, 2).double().cpu().numpy(), S.double().cpu().numpy()


@pytest.mark.parametrize("pairing", ["prefix", "same_step"])
@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_chain_matches_longer_prefill(F, variant, dtype, pairing):
    """prefill(L0) -> carry -> decode steps == oracle over L0 + steps tokens,
    under the prefix pair and the same-step pair (whose decode reads phi(k_t)
    itself and no x_prev)."""
    w = 4 if variant in ("F3", "F3A") else 1
    L0, steps = 70, 9
    d, outs, S = _decode_chain(F, variant, 3, 4, 64, 64, L0, steps, dtype, w, pairing=pairing)
    oo, oS = oracle_fwd(d, variant, w, pairing=pairing)
    tol = TOL[dtype]
    assert rel(outs, oo[:, :, L0:]) <= tol
    assert rel(S, oS) <= tol


@pytest.mark.parametrize("variant,dk,w,dtype", [("F2A", 128, 1, "bf16"), ("F2A", 128, 1, "f32"),
                                                ("F1", 64, 1, "bf16"), ("F3", 64, 4, "bf16"),
                                                ("F1", 64, 1, "f32")])
def test_decode_chain_4096_steps(F, variant, dk, w, dtype):
    """The decode length of the long-sequence workload: 4,096 decode steps
    after a 64-token prefill, fp32 state (N = 2, H = 2, lambda = 0.02).  Every
    step's output and the final state against the fp64 recurrence over all
    4,160 tokens: fp32 state drift over thousands of updates stays within the
    tolerance."""
    L0, steps = 64, 4096
    d, outs, S = _decode_chain(F, variant, 2, 2, dk, dk, L0, steps, dtype, w, seed=5050)
    oo, oS = oracle_fwd(d, variant, w)
    tol = TOL[dtype]
    eo, eS = rel(outs, oo[:, :, L0:]), rel(S, oS)
    # per-step check on a spread of steps, so that a late drift cannot hide behind early large outputs
    for t in (0, 1, 1023, 2047, 3071, steps - 1):
        assert rel(outs[:, :, t], oo[:, :, L0 + t]) <= tol, (t, rel(outs[:, :, t], oo[:, :, L0 + t]))
    assert eo <= tol and eS <= tol, (eo, eS)


@pytest.mark.parametrize("pairing", ["prefix", "same_step"])
def test_decode_workload5_shape(F, pairing):
    """N=64, H=16, 128x128 fp32 state: a few steps after a short prefill."""
    d, outs, S = _decode_chain(F, "F2A", 64, 16, 128, 128, 40, 4, "bf16", 1, pairing=pairing)
    oo, oS = oracle_fwd(d, "F2A", 1, pairing=pairing)
    assert rel(outs, oo[:, :, 40:]) <= 2e-2
    assert rel(S, oS) <= 2e-2


@pytest.mark.parametrize("variant", ["F1", "F2A"])
@pytest.mark.parametrize("dk,dv", [(16, 32), (32, 16), (128, 64)])
def test_decode_odd_pair_count(F, variant, dk, dv):
    """An odd number of (n, h) pairs leaves the last decode block one pair short."""
    d, outs, S = _decode_chain(F, variant, 3, 3, dk, dv, 20, 5, "f32", 1)
    oo, oS = oracle_fwd(d, variant, 1)
    assert rel(outs, oo[:, :, 20:]) <= 1e-4
    assert rel(S, oS) <= 1e-4


@pytest.mark.parametrize("pairing", ["prefix", "same_step"])
@pytest.mark.parametrize("variant,w,dk,dv,dtype", [("F3", 2, 64, 64, "f32"), ("F3A", 3, 32, 16, "f32"),
                                                   ("F3", 4, 128, 128, "bf16"), ("F3A", 4, 16, 32, "bf16"),
                                                   ("F3", 5, 64, 32, "f32"), ("F3", 8, 32, 32, "f32")])
def test_decode_window_paths(F, variant, w, dk, dv, dtype, pairing):
    """The window decode kernels (windows 2-4 templated on the window, 5-8 the
    general one) at several widths, with 2 x 5 = 10 (n, h) pairs: the last
    block of four is half full."""
    d, outs, S = _decode_chain(F, variant, 2, 5, dk, dv, 30, 6, dtype, w, pairing=pairing)
    oo, oS = oracle_fwd(d, variant, w, pairing=pairing)
    tol = TOL[dtype]
    assert rel(outs, oo[:, :, 30:]) <= tol
    assert rel(S, oS) <= tol


@pytest.mark.parametrize("N,H", [(2, 5), (1, 4), (3, 1)])
def test_decode_d128_pair_counts(F, N, H):
    """d = 128 decode blocks take three (n, h) pairs: 10, 4 and 3 pairs."""
    d, outs, S = _decode_chain(F, "F2A", N, H, 128, 128, 20, 5, "f32", 1)
    oo, oS = oracle_fwd(d, "F2A", 1)
    assert rel(outs, oo[:, :, 20:]) <= 1e-4
    assert rel(S, oS) <= 1e-4


@pytest.mark.parametrize("variant", ["F1", "F2A"])
def test_decode_d128_state_16_byte_aligned(F, variant):
    """d = 128 decode on a state that is only 16-byte aligned (a view into a
    larger buffer) and on an aligned one, both against the fp64 recurrence
    after the same prefill: the row accesses need 16-byte alignment only."""
    N, H, dk, L0, steps = 2, 3, 128, 20, 5
    d = gen.draw(variant, N, H, L0 + steps, dk, dk, seed=606, dtype="f32", lam=0.02)
    pre = {n: d[n][:, :, :L0].contiguous() for n in ("q", "k", "v", "beta")}
    _, S = F.fwd(variant, "chunk", *(pre[n].cuda() for n in ("q", "k", "v", "beta")), d["lam"].cuda(), d["eps"],
                 chunk=64)
    oo, oS = oracle_fwd(d, variant, 1)
    tok = {n: d[n][:, :, L0:].movedim(2, 0).contiguous().cuda() for n in ("q", "k", "v", "beta")}
    for shift in (0, 4):  # floats: 0 keeps torch's alignment, 4 leaves 16 bytes
        buf = torch.zeros(S.numel() + 8, dtype=torch.float32, device="cuda")
        Sx = buf[shift:shift + S.numel()].view(S.shape)
        Sx.copy_(S)
        assert (Sx.data_ptr() % 32 == 0) == (shift == 0)
        x_prev, _ = F.carry_from_prefill(variant, pre["k"].cuda(), pre["v"].cuda(), 1)
        outs = torch.empty((steps, N, H, dk), dtype=torch.float32, device="cuda")
        for i in range(steps):
            F.decode_step(variant, tok["q"][i], tok["k"][i], tok["v"][i], tok["beta"][i], d["lam"].cuda(), d["eps"],
                          1, Sx, x_prev, None, out=outs[i])
        torch.cuda.synchronize()
        o = outs.movedim(0, 2).double().cpu().numpy()
        assert rel(o, oo[:, :, L0:]) <= 1e-4, shift
        assert rel(Sx.double().cpu().numpy(), oS) <= 1e-4, shift


# --------------------------------------------------------------- tensor-core path options and extremes

@pytest.mark.parametrize("pairing,phi", [("same_step", "l2"), ("prefix", "identity"), ("same_step", "identity")])
@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_tensor_core_pairing_and_feature_map(F, variant, pairing, phi):
    """bf16, d = 64, chunk 64: the tensor-core chunk path with the same-step
    pair and the identity feature map."""
    d = gen.draw(variant, 2, 3, 150, 64, 64, seed=61, dtype="bf16", key_scale=0.125)
    check(F, d, variant, "chunk", chunk=64, pairing=pairing, phi=phi)


@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_tensor_core_strong_forgetting(F, variant):
    """lambda = 0.999 on the tensor-core path: chunk log-decays around -45, so
    the factorised decays use factors up to about e^22."""
    d = gen.draw(variant, 1, 4, 200, 64, 64, seed=62, dtype="bf16", lam=0.999)
    check(F, d, variant, "chunk", chunk=64)


@pytest.mark.parametrize("variant", ["F1", "F1A"])
def test_tensor_core_decay_floor(F, variant):
    """Tiny keys under the identity map with lambda = 0.9 put every alpha on
    the 2^-20 floor: a chunk's log-decay is near -887, far below -80, so every
    decay factor is taken as one exponential of a difference."""
    d = gen.draw(variant, 1, 4, 200, 64, 64, seed=63, dtype="bf16", lam=0.9, key_scale=0.05)
    check(F, d, variant, "chunk", chunk=64, phi="identity")


# --------------------------------------------------------------- the per-channel (Falcon-2A, d = 128) tensor-core path

@pytest.mark.parametrize("L", [64, 200, 513])
def test_falcon2a_d128_tensor_core_path(F, L):
    """bf16 Falcon-2A, d_k = d_v = 128, chunk 64: dS per chunk, the state scan
    and the outputs on tcgen05; one chunk, a ragged tail, many chunks."""
    d = gen.draw("F2A", 2, 3, L, 128, 128, seed=70 + L, dtype="bf16", lam=0.02)
    check(F, d, "F2A", "chunk", chunk=64)


@pytest.mark.parametrize("pairing,phi", [("same_step", "l2"), ("prefix", "identity")])
def test_falcon2a_d128_pairing_and_feature_map(F, pairing, phi):
    d = gen.draw("F2A", 1, 2, 150, 128, 128, seed=74, dtype="bf16", key_scale=0.09)
    check(F, d, "F2A", "chunk", chunk=64, pairing=pairing, phi=phi)


def test_falcon2a_d128_strong_forgetting(F):
    """lambda = 0.999: per-channel chunk log-decays around -45; factorised."""
    d = gen.draw("F2A", 1, 3, 200, 128, 128, seed=75, dtype="bf16", lam=0.999)
    check(F, d, "F2A", "chunk", chunk=64)


def test_falcon2a_d128_decay_floor(F):
    """Tiny keys under the identity map with lambda = 0.9: alpha sits on the
    2^-20 floor, the chunk log-decay is far below -80 and every intra-chunk
    decay factor is one exponential of a difference."""
    d = gen.draw("F2A", 1, 2, 130, 128, 128, seed=76, dtype="bf16", lam=0.9, key_scale=0.03)
    check(F, d, "F2A", "chunk", chunk=64, phi="identity")


# --------------------------------------------------------------- the per-channel regression (Falcon-2, d = 128) tensor-core path

@pytest.mark.parametrize("L", [64, 200, 513])
def test_falcon2_d128_tensor_core_path(F, L):
    """bf16 Falcon-2, d_k = d_v = 128, chunk 64: two blocks of 64 channels
    per head, the per-channel systems by forward substitution, the products
    on tcgen05; one chunk, a ragged tail, many chunks."""
    d = gen.draw("F2", 2, 3, L, 128, 128, seed=80 + L, dtype="bf16", lam=0.02)
    check(F, d, "F2", "chunk", chunk=64)


@pytest.mark.parametrize("pairing,phi", [("same_step", "l2"), ("prefix", "identity")])
def test_falcon2_d128_pairing_and_feature_map(F, pairing, phi):
    d = gen.draw("F2", 1, 2, 150, 128, 128, seed=84, dtype="bf16", key_scale=0.09)
    check(F, d, "F2", "chunk", chunk=64, pairing=pairing, phi=phi)


def test_falcon2_d128_strong_forgetting(F):
    """lambda = 0.999: per-channel chunk log-decays around -45, inside the
    range of the factorised outputs."""
    d = gen.draw("F2", 1, 3, 200, 128, 128, seed=85, dtype="bf16", lam=0.999)
    check(F, d, "F2", "chunk", chunk=64)


def test_falcon2_d128_decay_floor(F):
    """Tiny keys under the identity map with lambda = 0.9: alpha sits on the
    2^-20 floor, the chunk log-decay is far below -80, and the block solves
    for eta E with one exponential per term."""
    d = gen.draw("F2", 1, 2, 130, 128, 128, seed=86, dtype="bf16", lam=0.9, key_scale=0.03)
    check(F, d, "F2", "chunk", chunk=64, phi="identity")


@pytest.mark.parametrize("lam,key_scale,phi", [(0.02, 1.0, "l2"), (0.9, 0.03, "identity")])
def test_falcon2_d128_one_block_per_head(F, lam, key_scale, phi):
    """B*H = 80 heads: twice that many blocks would not fit on the SMs at
    once, so each head runs as one block over all 128 channels (two threads
    per channel in the solve) instead of two blocks of 64 channels; with and
    without the decay floor."""
    d = gen.draw("F2", 5, 16, 130, 128, 128, seed=87, dtype="bf16", lam=lam, key_scale=key_scale)
    check(F, d, "F2", "chunk", chunk=64, phi=phi)


# --------------------------------------------------------------- the windowed (Falcon-3/3A, d = 64) tensor-core path

@pytest.mark.parametrize("w", [2, 3, 4])
@pytest.mark.parametrize("variant", ["F3", "F3A"])
@pytest.mark.parametrize("L", [1, 5, 64, 65, 200])
def test_window_tensor_core_path(F, variant, w, L):
    """bf16 Falcon-3/3A, d_k = d_v = 64, chunk 64: per-chunk images written
    for the chain kernel (Falcon-3: the windowed system walked for the value
    channels and the rows of the identity, Falcon-3A: for the value channels
    alone); the products on tcgen05; one chunk and a ragged tail over several
    chunks."""
    d = gen.draw(variant, 2, 3, L, 64, 64, seed=100 + 10 * w + L, dtype="bf16")
    check(F, d, variant, "chunk", chunk=64, window=w)


@pytest.mark.parametrize("variant", ["F3", "F3A"])
def test_window_tensor_core_strong_forgetting(F, variant):
    """lambda = 0.999 with a window of 4: chunk log-decays far below zero but
    above -80, inside the factorised form."""
    d = gen.draw(variant, 1, 3, 200, 64, 64, seed=131, dtype="bf16", lam=0.999)
    check(F, d, variant, "chunk", chunk=64, window=4)


@pytest.mark.parametrize("w", [2, 3, 4])
@pytest.mark.parametrize("variant", ["F3", "F3A"])
def test_window_tensor_core_decay_floor(F, variant, w):
    """Tiny keys under the identity map with lambda = 0.9: alpha on the 2^-20
    floor, chunk log-decays far below -80; those chunks run the recurrence
    token by token on the value channels and the identity rows (Falcon-3),
    or sum their intra-chunk outputs with one exponential per term
    (Falcon-3A)."""
    d = gen.draw(variant, 1, 2, 150, 64, 64, seed=132 + w, dtype="bf16", lam=0.9, key_scale=0.03)
    check(F, d, variant, "chunk", chunk=64, window=w, phi="identity")


@pytest.mark.parametrize("pairing,phi", [("same_step", "l2"), ("prefix", "identity")])
@pytest.mark.parametrize("variant", ["F3", "F3A"])
def test_window_tensor_core_pairing_and_feature_map(F, variant, pairing, phi):
    d = gen.draw(variant, 1, 2, 150, 64, 64, seed=133, dtype="bf16", key_scale=0.2)
    check(F, d, variant, "chunk", chunk=64, window=4, pairing=pairing, phi=phi)
