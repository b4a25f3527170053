"""The C-ABI library loads and exports every symbol include/falcon.h declares;
argument validation answers with the documented codes before touching the
GPU (no compute call is made here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from linear_attention_sequence_falcon_b200 import build
    build.build()
    from linear_attention_sequence_falcon_b200 import _lib
    return _lib.load()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names.update(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(falcon_\w+)\s*\(", src, flags=re.M))
    return names


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert {"falcon_fwd", "falcon_fwd_ex", "falcon_decode_step", "falcon_decode_carry_from_prefill",
            "falcon_status_string"} <= names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -6, -7, -8, -9, 12345):
        s = lib.falcon_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0


def _fwd(lib, variant=0, form=2, dtype=1, window=1, B=1, H=1, L=8, dk=64, dv=64, chunk=64, ptr=1):
    P = ctypes.c_void_p(ptr) if ptr else None
    return lib.falcon_fwd(variant, form, dtype, P, P, P, P, P, 1e-6, window, B, H, L, dk, dv, chunk, P, P, None)


def test_validation_codes(lib):
    assert _fwd(lib, variant=6) == -2
    assert _fwd(lib, form=3) == -2
    assert _fwd(lib, dtype=7) == -2
    assert _fwd(lib, dk=48) == -3
    assert _fwd(lib, dv=256) == -3
    assert _fwd(lib, L=-1) == -3
    assert _fwd(lib, chunk=100) == -4
    assert _fwd(lib, chunk=128, variant=1) == -4          # chunk 128: Falcon-1/1A only,
    assert _fwd(lib, chunk=128, dtype=0) == -4            # with bf16 inputs
    assert _fwd(lib, chunk=128, dk=128, dv=128) == -4     # and d = 32 or 64
    assert _fwd(lib, chunk=128, dk=32, dv=64) == -4
    assert _fwd(lib, chunk=256) == -4
    assert _fwd(lib, variant=2, window=0) == -6
    assert _fwd(lib, variant=5, window=9) == -6
    assert _fwd(lib, ptr=0) == -1
    # empty batch: nothing to do, nothing enqueued
    assert _fwd(lib, B=0) == 0
    P = ctypes.c_void_p(1)
    assert lib.falcon_decode_step(2, 1, P, P, P, P, P, 1e-6, 3, 4, 2, 64, 64, P, P, None, P, None) == -1
    assert lib.falcon_decode_step(0, 1, P, P, P, P, P, 1e-6, 1, 4, 2, 64, 100, P, P, None, P, None) == -3
    assert lib.falcon_decode_carry_from_prefill(9, 1, P, P, 1, 1, 1, 4, 64, 64, P, None, None) == -2
    assert lib.falcon_decode_carry_from_prefill(2, 1, P, P, 4, 1, 1, 4, 64, 64, P, None, None) == -1


def _bwd(lib, variant=3, dtype=1, pairing=0, phi=0, window=1, B=1, H=1, L=8, dk=64, dv=64, ptr=1, dlam=True):
    P = ctypes.c_void_p(ptr) if ptr else None
    return lib.falcon_bwd(variant, dtype, pairing, phi, P, P, P, P, P, 1e-6, window, B, H, L, dk, dv, P, None,
                          P, P, P, P, P if dlam else None, None)


def test_backward_validation_codes(lib):
    lib.falcon_bwd.restype = ctypes.c_int
    assert _bwd(lib, variant=9) == -2
    assert _bwd(lib, dtype=4) == -2
    assert _bwd(lib, pairing=2) == -2
    assert _bwd(lib, phi=3) == -2
    assert _bwd(lib, dk=48) == -3
    assert _bwd(lib, variant=2, window=0) == -6
    assert _bwd(lib, variant=5, window=9) == -6
    assert _bwd(lib, dk=64, dv=32) == -9
    assert _bwd(lib, dk=16, dv=16) == -9
    assert _bwd(lib, ptr=0) == -1
    assert _bwd(lib, B=0) == 0
    assert _bwd(lib, L=0, dlam=False) == 0


def _host(lib, variants=(0, 3), form=2, dtype=1, window=1, B=1, H=1, L=8, dk=64, dv=64, chunk=64, ptr=1,
          outs=(1, 1), slices=0, vnull=False):
    P = ctypes.c_void_p(ptr) if ptr else None
    n = len(variants)
    vids = None if vnull else (ctypes.c_int * max(n, 1))(*variants)
    out = (ctypes.c_void_p * max(len(outs), 1))(*outs)
    return lib.falcon_fwd_host(n, vids, form, dtype, 0, 0, P, P, P, P, P, 1e-6, window, B, H, L, dk, dv, chunk,
                               out, None, slices, None)


def test_host_validation_codes(lib):
    """falcon_fwd_host answers argument errors before any copy or launch."""
    lib.falcon_fwd_host.restype = ctypes.c_int
    assert _host(lib, variants=()) == -9
    assert _host(lib, variants=(0,) * 7, outs=(1,) * 7) == -9
    assert _host(lib, slices=-1) == -9
    assert _host(lib, vnull=True) == -1
    assert _host(lib, variants=(0, 9)) == -2
    assert _host(lib, variants=(0, 1)) == -9  # scalar and per-channel beta in one call
    assert _host(lib, variants=(1, 4), B=0) == 0  # Falcon-2 and Falcon-2A share the per-channel layout
    assert _host(lib, chunk=100) == -4
    assert _host(lib, dk=48) == -3
    assert _host(lib, variants=(2,), outs=(1,), window=0) == -6
    assert _host(lib, ptr=0) == -1
    assert _host(lib, outs=(1, 0)) == -1
    assert _host(lib, B=0) == 0


# --------------------------------------------------------------- caller-owned workspace (no library allocation)

def _size(lib, variant=0, form=2, dtype=1, pairing=0, phi=0, window=1, B=8, H=12, L=2048, dk=64, dv=64, chunk=64):
    n = ctypes.c_size_t(12345)
    rc = lib.falcon_fwd_workspace_size(variant, form, dtype, pairing, phi, window, B, H, L, dk, dv, chunk,
                                       ctypes.byref(n))
    return rc, n.value


def test_workspace_size_query(lib):
    """The size query is host-only: the tensor-core chunk paths and the masked
    form need a workspace, every other path none."""
    lib.falcon_fwd_workspace_size.restype = ctypes.c_int
    units = 8 * 12 * 32
    assert _size(lib) == (0, units * 32 * 1024 + units * 4)          # Falcon-1 chunk, bf16, d = 64
    assert _size(lib, variant=3) == (0, units * 32 * 1024 + units * 4)  # Falcon-1A
    assert _size(lib, dtype=0) == (0, 0)                              # fp32: the span kernel, no workspace
    assert _size(lib, chunk=32) == (0, 0)
    assert _size(lib, variant=1, B=4, H=16, L=4096, dk=128, dv=128) == (0, 0)  # Falcon-2: one block per head
    assert _size(lib, variant=4, B=2, H=16, L=32768, dk=128, dv=128)[1] == 2 * 16 * 512 * 98816  # Falcon-2A
    # masked: B*H*L*(window*dv + 2*dv) floats
    assert _size(lib, form=1, variant=2, window=4, B=2, H=3, L=100, dk=32, dv=32) == (0, 4 * 2 * 3 * 100 * 6 * 32)
    assert _size(lib, form=0) == (0, 0)
    assert _size(lib, L=0) == (0, 0)
    assert _size(lib, chunk=100) == (-4, 0)
    assert _size(lib, variant=7) == (-2, 0)
    assert lib.falcon_fwd_workspace_size(0, 2, 1, 0, 0, 1, 1, 1, 1, 64, 64, 64, None) == -1


def test_workspace_entry_points_refuse_bad_workspace(lib):
    """falcon_fwd_ws / falcon_bwd_ws / falcon_fwd_host_ws return
    FALCON_ERR_WORKSPACE (-11) for a missing, short or misaligned workspace,
    before anything is enqueued."""
    P = ctypes.c_void_p(0x1000)
    lib.falcon_fwd_ws.restype = ctypes.c_int
    _, need = _size(lib, B=1, H=1, L=128)
    args = (0, 2, 1, 0, 0, P, P, P, P, P, 1e-6, 1, 1, 1, 128, 64, 64, 64, None, None, None, P, P)
    assert lib.falcon_fwd_ws(*args, None, 0, None) == -11
    assert lib.falcon_fwd_ws(*args, ctypes.c_void_p(0x10000), need - 1, None) == -11
    assert lib.falcon_fwd_ws(*args, ctypes.c_void_p(0x10000 + 16), need, None) == -11  # not 256-byte aligned
    assert lib.falcon_status_string(-11) != b"unknown status"
    # the masked form too
    margs = (0, 1, 1, 0, 0, P, P, P, P, P, 1e-6, 1, 1, 1, 128, 64, 64, 64, None, None, None, P, P)
    assert lib.falcon_fwd_ws(*margs, None, 0, None) == -11
    # the backward
    lib.falcon_bwd_ws.restype = ctypes.c_int
    n = ctypes.c_size_t(0)
    for form in (0, 2):  # recurrent, chunk-parallel
        assert lib.falcon_bwd_workspace_size(0, form, 1, 0, 0, 1, 1, 1, 64, 64, 64, 64, ctypes.byref(n)) == 0
        assert n.value > 0
        assert lib.falcon_bwd_ws(0, form, 1, 0, 0, P, P, P, P, P, 1e-6, 1, 1, 1, 64, 64, 64, 64, P, None, P, P, P, P,
                                 None, ctypes.c_void_p(0x10000), n.value - 4, None) == -11

    # the host-buffer forward
    vids = (ctypes.c_int * 2)(0, 3)
    out = (ctypes.c_void_p * 2)(1, 1)
    hn = ctypes.c_size_t(0)
    assert lib.falcon_fwd_host_workspace_size(2, vids, 2, 1, 0, 0, 1, 2, 3, 128, 64, 64, 64, 0, 0,
                                              ctypes.byref(hn)) == 0
    assert hn.value > 0
    lib.falcon_fwd_host_ws.restype = ctypes.c_int
    assert lib.falcon_fwd_host_ws(2, vids, 2, 1, 0, 0, P, P, P, P, P, 1e-6, 1, 2, 3, 128, 64, 64, 64, out, None, 0,
                                  ctypes.c_void_p(0x10000), hn.value - 256, None) == -11


def test_same_step_decode_and_carry_validation(lib):
    """The same-step pair needs no x_prev in decode and carry; the prefix pair
    still does; unknown pairings are refused."""
    P = ctypes.c_void_p(1)
    lib.falcon_decode_step_ex.restype = ctypes.c_int
    assert lib.falcon_decode_step_ex(0, 1, 2, P, P, P, P, P, 1e-6, 1, 4, 2, 64, 64, P, P, None, P, None) == -2
    assert lib.falcon_decode_step_ex(0, 1, 0, P, P, P, P, P, 1e-6, 1, 4, 2, 64, 64, P, None, None, P, None) == -1
    assert lib.falcon_decode_step_ex(2, 1, 1, P, P, P, P, P, 1e-6, 3, 4, 2, 64, 64, P, None, None, P, None) == -1
    assert lib.falcon_decode_step_ex(0, 1, 1, P, P, P, P, P, 1e-6, 1, 0, 2, 64, 64, P, None, None, P, None) == 0
    lib.falcon_decode_carry_from_prefill_ex.restype = ctypes.c_int
    assert lib.falcon_decode_carry_from_prefill_ex(0, 1, 3, P, P, 1, 1, 1, 4, 64, 64, P, None, None) == -2
    assert lib.falcon_decode_carry_from_prefill_ex(0, 1, 0, P, P, 1, 1, 1, 4, 64, 64, None, None, None) == -1
    # same-step, no window, no x_prev: nothing to carry, nothing enqueued
    assert lib.falcon_decode_carry_from_prefill_ex(0, 1, 1, P, P, 1, 1, 1, 4, 64, 64, None, None, None) == 0


# --------------------------------------------------------------- binding shape checks (before any pointer is used)

def _cpu(*shape, dtype=None):
    import torch
    return torch.zeros(shape, dtype=dtype or torch.bfloat16)


def test_binding_checks_forward_shapes():
    import torch
    import linear_attention_sequence_falcon_b200 as F
    q = _cpu(2, 3, 10, 64)
    lam = torch.zeros(3)
    b1, b2 = _cpu(2, 3, 10), _cpu(2, 3, 10, 32)
    v = _cpu(2, 3, 10, 32)
    ok = F.check_fwd_shapes("F1", q, q, v, b1, lam)
    assert ok == (2, 3, 10, 64, 32)
    assert F.check_fwd_shapes("F2", q, q, v, b2, lam) == ok
    bad = [
        dict(variant="F1", k=_cpu(2, 3, 11, 64)),                 # k's L differs from q's
        dict(variant="F1", v=_cpu(2, 4, 10, 32)),                 # v's H differs
        dict(variant="F2", beta=b1),                              # Falcon-2 needs beta per value channel
        dict(variant="F1", beta=b2),                              # Falcon-1 takes one beta per token
        dict(variant="F1", lam=torch.zeros(4)),                   # lambda must have H entries
        dict(variant="F1", out=_cpu(2, 3, 10, 64)),               # out must be [B,H,L,d_v]
        dict(variant="F1", final_state=torch.zeros(2, 3, 64, 64)),  # state must be [B,H,d_v,d_k]
        dict(variant="F1", initial_state=torch.zeros(2, 3, 32, 32)),
        dict(variant="F1", x_prev=torch.zeros(2, 3, 32)),
        dict(variant="F3", window=4, win=torch.zeros(2, 3, 2, 96)),  # window-1 = 3 slots of d_k + d_v
        dict(variant="F9"),
    ]
    for case in bad:
        a = dict(variant="F1", q=q, k=q, v=v, beta=b1, lam=lam)
        a.update(case)
        variant = a.pop("variant")
        with pytest.raises(F.FalconError):
            F.check_fwd_shapes(variant, **a)
    # and through the public call, before any pointer reaches the library
    with pytest.raises(F.FalconError, match="shape"):
        F.fwd("F2", "chunk", q, q, v, b1, lam, 1e-6)
    with pytest.raises(F.FalconError, match="shape"):
        F.fwd("F1", "chunk", q, q, v, b1, torch.zeros(5), 1e-6)
    with pytest.raises(F.FalconError, match="shape"):
        F.bwd("F1", q, q, v, b1, lam, 1e-6, dout=_cpu(2, 3, 10, 64))


def test_binding_checks_decode_shapes():
    import torch
    import linear_attention_sequence_falcon_b200 as F
    q = _cpu(4, 2, 64)
    v = _cpu(4, 2, 64)
    lam = torch.zeros(2)
    st, xp = torch.zeros(4, 2, 64, 64), torch.zeros(4, 2, 64)
    assert F.check_decode_shapes("F1", q, q, v, _cpu(4, 2), lam, 1, st, xp, None) == (4, 2, 64, 64)
    with pytest.raises(F.FalconError):
        F.check_decode_shapes("F2A", q, q, v, _cpu(4, 2), lam, 1, st, xp, None)   # per-channel beta
    with pytest.raises(F.FalconError):
        F.check_decode_shapes("F1", q, q, v, _cpu(4, 2), lam, 1, torch.zeros(4, 2, 64, 32), xp, None)
    with pytest.raises(F.FalconError):
        F.check_decode_shapes("F3", q, q, v, _cpu(4, 2), lam, 4, st, xp, None)     # window carry missing
    with pytest.raises(F.FalconError):
        F.check_decode_shapes("F3", q, q, v, _cpu(4, 2), lam, 4, st, xp, torch.zeros(4, 2, 3, 64))
    with pytest.raises(F.FalconError):
        F.decode_step("F1", q, q, v, _cpu(4, 2), torch.zeros(3), 1e-6, 1, st, xp)


def test_chunk_backward_scope(lib):
    """The chunk-parallel backward takes Falcon-1/1A, bf16, d = 64, chunk 64;
    other requests are refused before anything is enqueued."""
    n = ctypes.c_size_t(0)
    size = lambda v, form, dt, d, ch: lib.falcon_bwd_workspace_size(v, form, dt, 0, 0, 1, 2, 3, 200, d, d, ch,
                                                                    ctypes.byref(n))
    assert size(0, 2, 1, 64, 64) == 0 and size(3, 2, 1, 64, 64) == 0
    assert size(1, 2, 1, 64, 64) == -9     # Falcon-2: recurrent form only
    assert size(0, 2, 0, 64, 64) == -9     # fp32 inputs
    assert size(0, 2, 1, 128, 64) == -9    # d = 128
    assert size(0, 2, 1, 64, 32) == -4     # chunk 32
    assert size(0, 1, 1, 64, 64) == -9     # masked form
    assert size(0, 7, 1, 64, 64) == -2
