"""ctypes binding of libfalcon.so (the C ABI declared in include/falcon.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  Tensors must already live on the GPU; the calls
enqueue on torch's current stream (or the stream given) and return without
synchronising.  There is no CPU fallback: if the library is missing or the
device is not a CUDA GPU, the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfalcon.so")

VARIANTS = {"F1": 0, "F2": 1, "F3": 2, "F1A": 3, "F2A": 4, "F3A": 5}
FORMS = {"recurrent": 0, "masked": 1, "chunk": 2}
DTYPES = {torch.float32: 0, torch.bfloat16: 1}
PAIRINGS = {"prefix": 0, "same_step": 1}
PHIS = {"l2": 0, "identity": 1}
EXPORTS = ("falcon_fwd", "falcon_fwd_ex", "falcon_fwd_host", "falcon_fwd_carry", "falcon_bwd", "falcon_decode_step", "falcon_decode_carry_from_prefill",
           "falcon_fwd_masked_noalloc", "falcon_device_wait_timeouts", "falcon_selftest_bounded_wait",
           "falcon_scratch_trim", "falcon_status_string")

_lib = None


class FalconError(RuntimeError):
    pass


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfalcon.so and declare the C signatures (raises if absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FalconError("libfalcon.so not built (run python -m linear_attention_sequence_falcon_b200.build)")
    lib = ctypes.CDLL(path)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.falcon_fwd.argtypes = [I, I, I, P, P, P, P, P, F, I, I, I, I, I, I, I, P, P, P]
    lib.falcon_fwd.restype = I
    lib.falcon_fwd_ex.argtypes = [I, I, I, I, I, P, P, P, P, P, F, I, I, I, I, I, I, I, P, P, P]
    lib.falcon_fwd_ex.restype = I
    lib.falcon_fwd_host.argtypes = [I, P, I, I, I, I, P, P, P, P, P, F, I, I, I, I, I, I, I, P, P, I, P]
    lib.falcon_fwd_host.restype = I
    lib.falcon_fwd_carry.argtypes = [I, I, I, P, P, P, P, P, F, I, I, I, I, I, I, I, P, P, P, P, P, P]
    lib.falcon_fwd_carry.restype = I
    lib.falcon_bwd.argtypes = [I, I, I, I, P, P, P, P, P, F, I, I, I, I, I, I, P, P, P, P, P, P, P, P]
    lib.falcon_bwd.restype = I
    lib.falcon_decode_step.argtypes = [I, I, P, P, P, P, P, F, I, I, I, I, I, P, P, P, P, P]
    lib.falcon_decode_step.restype = I
    lib.falcon_decode_carry_from_prefill.argtypes = [I, I, P, P, I, I, I, I, I, I, P, P, P]
    lib.falcon_decode_carry_from_prefill.restype = I
    lib.falcon_fwd_masked_noalloc.argtypes = [I, I, P, P, P, P, P, F, I, I, I, I, I, I, P, P, P]
    lib.falcon_fwd_masked_noalloc.restype = I
    lib.falcon_device_wait_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint)]
    lib.falcon_device_wait_timeouts.restype = I
    lib.falcon_selftest_bounded_wait.argtypes = [ctypes.c_uint, ctypes.POINTER(ctypes.c_int)]
    lib.falcon_selftest_bounded_wait.restype = I
    lib.falcon_scratch_trim.argtypes = []
    lib.falcon_scratch_trim.restype = I
    lib.falcon_status_string.argtypes = [I]
    lib.falcon_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(rc: int):
    if rc != 0:
        msg = load().falcon_status_string(rc).decode()
        raise FalconError("libfalcon status %d: %s" % (rc, msg))


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise FalconError("tensor is not on a CUDA device (no CPU path exists)")
    if not t.is_contiguous():
        raise FalconError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def fwd(variant: str, form: str, q, k, v, beta, lam, eps: float, window: int = 1, chunk: int = 64,
        out=None, final_state=None, pairing: str = "prefix", phi: str = "l2", stream=None,
        want_state: bool = True, initial_state=None, x_prev=None, win=None):
    """falcon_fwd_ex on CUDA tensors q,k [B,H,L,dk], v [B,H,L,dv], beta [B,H,L] or
    [B,H,L,dv] (same dtype), lam [H] fp32.  Returns (out, final_state).
    With initial_state [B,H,dv,dk], x_prev [B,H,dk] or win [B,H,window-1,dk+dv]
    (fp32; the decode carry) it is falcon_fwd_carry: a segment continuing a
    sequence (prefix pairing, L2 feature map)."""
    lib = load()
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    if q.dtype not in DTYPES or not (q.dtype == k.dtype == v.dtype == beta.dtype):
        raise FalconError("q, k, v, beta must share one dtype, fp32 or bf16")
    if lam.dtype != torch.float32:
        raise FalconError("lambda must be fp32")
    if out is None:
        out = torch.empty((B, H, L, dv), dtype=q.dtype, device=q.device)
    if final_state is None and want_state:
        final_state = torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device)
    carry = (initial_state, x_prev, win)
    if any(c is not None for c in carry):
        if pairing != "prefix" or phi != "l2":
            raise FalconError("a continued segment uses the prefix pairing and the L2 feature map")
        for c in carry:
            if c is not None and (c.dtype != torch.float32 or not c.is_contiguous()):
                raise FalconError("initial_state, x_prev and win must be contiguous fp32")
        rc = lib.falcon_fwd_carry(VARIANTS[variant], FORMS[form], DTYPES[q.dtype],
                                  _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(lam), float(eps), int(window),
                                  B, H, L, dk, dv, int(chunk), *(_ptr(c) if c is not None else None for c in carry),
                                  _ptr(out), _ptr(final_state), _stream(stream))
    else:
        rc = lib.falcon_fwd_ex(VARIANTS[variant], FORMS[form], DTYPES[q.dtype], PAIRINGS[pairing], PHIS[phi],
                               _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(lam), float(eps), int(window),
                               B, H, L, dk, dv, int(chunk), _ptr(out), _ptr(final_state), _stream(stream))
    _check(rc)
    return out, final_state


def _host_ptr(t):
    if t is None:
        return None
    if t.is_cuda:
        raise FalconError("fwd_host takes host (CPU) tensors")
    if not t.is_contiguous():
        raise FalconError("tensor must be contiguous")
    return t.data_ptr()


def fwd_host(variants, form: str, q, k, v, beta, lam, eps: float, window: int = 1, chunk: int = 64,
             out=None, final_state=None, pairing: str = "prefix", phi: str = "l2", slices: int = 0,
             want_state: bool = True, stream=None):
    """falcon_fwd_host: the forward of one or several variants over the same
    inputs in host memory (CPU tensors; pinned memory lets the library overlap
    the copies of one batch slice with the compute of the next).  q,k
    [B,H,L,dk], v [B,H,L,dv], beta [B,H,L] or [B,H,L,dv] (same dtype), lam [H]
    fp32.  Returns (outs, states): lists of CPU tensors, one per variant
    (pinned when allocated here).  The call only enqueues; synchronise the
    stream before reading the results."""
    lib = load()
    if isinstance(variants, str):
        variants = [variants]
    n = len(variants)
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    if q.dtype not in DTYPES or not (q.dtype == k.dtype == v.dtype == beta.dtype):
        raise FalconError("q, k, v, beta must share one dtype, fp32 or bf16")
    if lam.dtype != torch.float32:
        raise FalconError("lambda must be fp32")
    pin = torch.cuda.is_available()
    if out is None:
        out = [torch.empty((B, H, L, dv), dtype=q.dtype, pin_memory=pin) for _ in range(n)]
    if final_state is None and want_state:
        final_state = [torch.empty((B, H, dv, dk), dtype=torch.float32, pin_memory=pin) for _ in range(n)]
    if len(out) != n or (final_state is not None and len(final_state) != n):
        raise FalconError("one output (and one state) per variant")
    vids = (ctypes.c_int * n)(*(VARIANTS[x] for x in variants))
    outs = (ctypes.c_void_p * n)(*(_host_ptr(o) for o in out))
    states = None
    if final_state is not None:
        for st in final_state:
            if st is not None and st.dtype != torch.float32:
                raise FalconError("final states are fp32")
        states = (ctypes.c_void_p * n)(*(_host_ptr(st) for st in final_state))
    hp = lambda t: ctypes.c_void_p(_host_ptr(t))  # noqa: E731
    rc = lib.falcon_fwd_host(n, vids, FORMS[form], DTYPES[q.dtype], PAIRINGS[pairing], PHIS[phi],
                             hp(q), hp(k), hp(v), hp(beta), hp(lam), float(eps), int(window),
                             B, H, L, dk, dv, int(chunk), outs, states, int(slices), _stream(stream))
    _check(rc)
    return out, final_state


def bwd(variant: str, q, k, v, beta, lam, eps: float, dout, dstate=None, window: int = 1, pairing: str = "prefix",
        phi: str = "l2", stream=None):
    """falcon_bwd: gradients of a loss with respect to q, k, v, beta and lambda
    of a forward from S_0 = 0, given dout = dL/d(out) (dtype of q) and dstate =
    dL/d(final_state) (fp32, or None).  Every variant (window for Falcon-3/3A),
    d_k = d_v in {32, 64, 128}.  Returns a dict of fp32 tensors dq, dk, dv, dbeta, dlambda."""
    lib = load()
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    if q.dtype not in DTYPES or not (q.dtype == k.dtype == v.dtype == beta.dtype == dout.dtype):
        raise FalconError("q, k, v, beta, dout must share one dtype, fp32 or bf16")
    if lam.dtype != torch.float32 or (dstate is not None and dstate.dtype != torch.float32):
        raise FalconError("lambda and dstate must be fp32")
    f32 = dict(dtype=torch.float32, device=q.device)
    g = {"dq": torch.empty((B, H, L, dk), **f32), "dk": torch.empty((B, H, L, dk), **f32),
         "dv": torch.empty((B, H, L, dv), **f32), "dbeta": torch.empty(tuple(beta.shape), **f32),
         "dlambda": torch.zeros((H,), **f32)}
    rc = lib.falcon_bwd(VARIANTS[variant], DTYPES[q.dtype], PAIRINGS[pairing], PHIS[phi],
                        _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(lam), float(eps), int(window), B, H, L, dk, dv,
                        _ptr(dout), _ptr(dstate) if dstate is not None else None,
                        _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dbeta"]), _ptr(g["dlambda"]),
                        _stream(stream))
    _check(rc)
    return g


def fwd_masked_noalloc(variant: str, q, k, v, beta, lam, eps: float, window: int = 1, out=None,
                       final_state=None, stream=None):
    """falcon_fwd_masked_noalloc: the masked-parallel forward for callers that
    may not allocate device memory (a host that owns all device allocations,
    a fixed memory budget).  Its scratch is a fixed array inside the library;
    problems beyond it raise (FALCON_ERR_SCRATCH).  Calls sharing a device
    must not overlap on the GPU.  Same results as fwd(..., form="masked")."""
    lib = load()
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, H, L, dv), dtype=q.dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device)
    rc = lib.falcon_fwd_masked_noalloc(VARIANTS[variant], DTYPES[q.dtype], _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                       _ptr(lam), float(eps), int(window), B, H, L, dk, dv, _ptr(out),
                                       _ptr(final_state), _stream(stream))
    _check(rc)
    return out, final_state


def selftest_bounded_wait(timeout_us: int = 2000) -> int:
    """Runs the on-device bounded-wait check; returns 1 when the wait gave up."""
    r = ctypes.c_int(-1)
    _check(load().falcon_selftest_bounded_wait(int(timeout_us), ctypes.byref(r)))
    return int(r.value)


def scratch_trim() -> None:
    """Return the unused memory of the current device's scratch pool."""
    _check(load().falcon_scratch_trim())


def wait_timeouts() -> int:
    """Diagnostic counter of tensor-core thread blocks that gave up waiting."""
    c = ctypes.c_uint(0)
    _check(load().falcon_device_wait_timeouts(ctypes.byref(c)))
    return int(c.value)


def decode_step(variant: str, q, k, v, beta, lam, eps: float, window: int, state, x_prev, win=None,
                out=None, stream=None):
    """falcon_decode_step: q,k [N,H,dk], v [N,H,dv], beta [N,H] or [N,H,dv];
    state [N,H,dv,dk], x_prev [N,H,dk], win [N,H,window-1,dk+dv] fp32 (in/out)."""
    lib = load()
    N, H, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    rc = lib.falcon_decode_step(VARIANTS[variant], DTYPES[q.dtype], _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                _ptr(lam), float(eps), int(window), N, H, dk, dv, _ptr(state), _ptr(x_prev),
                                _ptr(win), _ptr(out), _stream(stream))
    _check(rc)
    return out


def carry_from_prefill(variant: str, k, v, window: int, x_prev=None, win=None, stream=None):
    """falcon_decode_carry_from_prefill: returns (x_prev [B,H,dk], win [B,H,w-1,dk+dv])."""
    lib = load()
    B, H, L, dk = k.shape
    dv = v.shape[-1]
    w = window if variant in ("F3", "F3A") else 1
    if x_prev is None:
        x_prev = torch.empty((B, H, dk), dtype=torch.float32, device=k.device)
    if win is None and w > 1:
        win = torch.empty((B, H, w - 1, dk + dv), dtype=torch.float32, device=k.device)
    rc = lib.falcon_decode_carry_from_prefill(VARIANTS[variant], DTYPES[k.dtype], _ptr(k), _ptr(v), int(window),
                                              B, H, L, dk, dv, _ptr(x_prev), _ptr(win), _stream(stream))
    _check(rc)
    return x_prev, win
