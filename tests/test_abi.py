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
    assert _fwd(lib, chunk=128) == -4
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
