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
EXPORTS = ("falcon_fwd", "falcon_fwd_ex", "falcon_fwd_workspace_size", "falcon_fwd_ws", "falcon_fwd_host",
           "falcon_fwd_host_workspace_size", "falcon_fwd_host_ws", "falcon_fwd_carry", "falcon_fwd_carry_ex",
           "falcon_bwd", "falcon_bwd_ex", "falcon_bwd_workspace_size", "falcon_bwd_ws", "falcon_decode_step",
           "falcon_decode_step_ex", "falcon_decode_carry_from_prefill", "falcon_decode_carry_from_prefill_ex",
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
    Z, ZP = ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t)
    lib.falcon_fwd_workspace_size.argtypes = [I, I, I, I, I, I, I, I, I, I, I, I, ZP]
    lib.falcon_fwd_workspace_size.restype = I
    lib.falcon_fwd_ws.argtypes = [I, I, I, I, I, P, P, P, P, P, F, I, I, I, I, I, I, I, P, P, P, P, P, P, Z, P]
    lib.falcon_fwd_ws.restype = I
    lib.falcon_fwd_host_workspace_size.argtypes = [I, P, I, I, I, I, I, I, I, I, I, I, I, I, I, ZP]
    lib.falcon_fwd_host_workspace_size.restype = I
    lib.falcon_fwd_host_ws.argtypes = [I, P, I, I, I, I, P, P, P, P, P, F, I, I, I, I, I, I, I, P, P, I, P, Z, P]
    lib.falcon_fwd_host_ws.restype = I
    lib.falcon_fwd_carry.argtypes = [I, I, I, P, P, P, P, P, F, I, I, I, I, I, I, I, P, P, P, P, P, P]
    lib.falcon_fwd_carry.restype = I
    lib.falcon_fwd_carry_ex.argtypes = [I, I, I, I, I, P, P, P, P, P, F, I, I, I, I, I, I, I, P, P, P, P, P, P]
    lib.falcon_fwd_carry_ex.restype = I
    lib.falcon_bwd.argtypes = [I, I, I, I, P, P, P, P, P, F, I, I, I, I, I, I, P, P, P, P, P, P, P, P]
    lib.falcon_bwd.restype = I
    lib.falcon_bwd_ex.argtypes = [I, I, I, I, I, P, P, P, P, P, F, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P]
    lib.falcon_bwd_ex.restype = I
    lib.falcon_bwd_workspace_size.argtypes = [I, I, I, I, I, I, I, I, I, I, I, I, ZP]
    lib.falcon_bwd_workspace_size.restype = I
    lib.falcon_bwd_ws.argtypes = [I, I, I, I, I, P, P, P, P, P, F, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, Z, P]
    lib.falcon_bwd_ws.restype = I
    lib.falcon_decode_step.argtypes = [I, I, P, P, P, P, P, F, I, I, I, I, I, P, P, P, P, P]
    lib.falcon_decode_step.restype = I
    lib.falcon_decode_step_ex.argtypes = [I, I, I, P, P, P, P, P, F, I, I, I, I, I, P, P, P, P, P]
    lib.falcon_decode_step_ex.restype = I
    lib.falcon_decode_carry_from_prefill.argtypes = [I, I, P, P, I, I, I, I, I, I, P, P, P]
    lib.falcon_decode_carry_from_prefill.restype = I
    lib.falcon_decode_carry_from_prefill_ex.argtypes = [I, I, I, P, P, I, I, I, I, I, I, P, P, P]
    lib.falcon_decode_carry_from_prefill_ex.restype = I
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


def _shape_error(msg):
    raise FalconError("shape: " + msg)


def _window(variant, window):
    return int(window) if variant in ("F3", "F3A") else 1


def check_fwd_shapes(variant, q, k, v, beta, lam, window=1, out=None, final_state=None, initial_state=None,
                     x_prev=None, win=None):
    """Checks every array of a forward against q's [B,H,L,d_k] before any
    pointer reaches the library (the C ABI cannot see sizes): k like q, v
    [B,H,L,d_v], beta [B,H,L] or [B,H,L,d_v] (Falcon-2/2A), lambda [H], out
    [B,H,L,d_v], final and initial states [B,H,d_v,d_k], x_prev [B,H,d_k],
    win [B,H,window-1,d_k+d_v]; all on one device.  Raises FalconError."""
    if variant not in VARIANTS:
        raise FalconError("unknown variant %r" % (variant,))
    if q.dim() != 4:
        _shape_error("q must be [B,H,L,d_k], got %s" % (tuple(q.shape),))
    B, H, L, dk = q.shape
    if tuple(k.shape) != (B, H, L, dk):
        _shape_error("k %s must match q %s" % (tuple(k.shape), tuple(q.shape)))
    if v.dim() != 4 or tuple(v.shape[:3]) != (B, H, L):
        _shape_error("v must be [B,H,L,d_v] with q's B,H,L, got %s" % (tuple(v.shape),))
    dv = v.shape[3]
    want = (B, H, L, dv) if variant in ("F2", "F2A") else (B, H, L)
    if tuple(beta.shape) != want:
        _shape_error("beta of %s must be %s, got %s" % (variant, want, tuple(beta.shape)))
    if tuple(lam.shape) != (H,):
        _shape_error("lambda must be [H] = (%d,), got %s" % (H, tuple(lam.shape)))
    w = _window(variant, window)
    checks = ((out, (B, H, L, dv), "out"), (final_state, (B, H, dv, dk), "final_state"),
              (initial_state, (B, H, dv, dk), "initial_state"), (x_prev, (B, H, dk), "x_prev"),
              (win, (B, H, w - 1, dk + dv), "win"))
    for t, shape, name in checks:
        if t is not None and tuple(t.shape) != shape:
            _shape_error("%s must be %s, got %s" % (name, shape, tuple(t.shape)))
    for t in (k, v, beta, lam, out, final_state, initial_state, x_prev, win):
        if t is not None and t.device != q.device:
            raise FalconError("every tensor must be on q's device (%s)" % (q.device,))
    return B, H, L, dk, dv


def _alloc_workspace(nbytes, device, stream):
    """Device workspace the caller (torch's allocator) owns, lent to one call."""
    if nbytes == 0:
        return None
    ws = torch.empty(int(nbytes), dtype=torch.uint8, device=device)
    if stream is not None and stream != torch.cuda.current_stream(device):
        ws.record_stream(stream)
    return ws


def fwd_workspace_size(variant: str, form: str, dtype, B: int, H: int, L: int, dk: int, dv: int, window: int = 1,
                       chunk: int = 64, pairing: str = "prefix", phi: str = "l2") -> int:
    """falcon_fwd_workspace_size: device bytes the forward with these shapes needs."""
    n = ctypes.c_size_t(0)
    _check(load().falcon_fwd_workspace_size(VARIANTS[variant], FORMS[form], DTYPES[dtype], PAIRINGS[pairing],
                                            PHIS[phi], int(window), B, H, L, dk, dv, int(chunk), ctypes.byref(n)))
    return int(n.value)


def fwd(variant: str, form: str, q, k, v, beta, lam, eps: float, window: int = 1, chunk: int = 64,
        out=None, final_state=None, pairing: str = "prefix", phi: str = "l2", stream=None,
        want_state: bool = True, initial_state=None, x_prev=None, win=None, workspace=None):
    """The forward on CUDA tensors q,k [B,H,L,dk], v [B,H,L,dv], beta [B,H,L]
    or [B,H,L,dv] (same dtype), lam [H] fp32.  Returns (out, final_state).
    With initial_state [B,H,dv,dk], x_prev [B,H,dk] or win [B,H,window-1,dk+dv]
    (fp32; the decode carry) the sequence continues an earlier segment.
    Runs through falcon_fwd_ws: the workspace (falcon_fwd_workspace_size
    bytes, when the path needs one) is `workspace` (a uint8 CUDA tensor) or
    drawn here from torch's allocator; the library allocates nothing."""
    lib = load()
    B, H, L, dk, dv = check_fwd_shapes(variant, q, k, v, beta, lam, window, out, final_state, initial_state,
                                       x_prev, win)
    if q.dtype not in DTYPES or not (q.dtype == k.dtype == v.dtype == beta.dtype):
        raise FalconError("q, k, v, beta must share one dtype, fp32 or bf16")
    if lam.dtype != torch.float32:
        raise FalconError("lambda must be fp32")
    if out is not None and out.dtype != q.dtype:
        raise FalconError("out must have q's dtype")
    for c in (final_state, initial_state, x_prev, win):
        if c is not None and c.dtype != torch.float32:
            raise FalconError("states, x_prev and win are fp32")
    if out is None:
        out = torch.empty((B, H, L, dv), dtype=q.dtype, device=q.device)
    if final_state is None and want_state:
        final_state = torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device)
    need = fwd_workspace_size(variant, form, q.dtype, B, H, L, dk, dv, window, chunk, pairing, phi)
    if workspace is None:
        workspace = _alloc_workspace(need, q.device, stream)
    elif workspace.numel() * workspace.element_size() < need:
        raise FalconError("workspace of %d bytes is smaller than the %d the call needs"
                          % (workspace.numel() * workspace.element_size(), need))
    wsp = _ptr(workspace) if workspace is not None else None
    wsn = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.falcon_fwd_ws(VARIANTS[variant], FORMS[form], DTYPES[q.dtype], PAIRINGS[pairing], PHIS[phi],
                           _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(lam), float(eps), int(window),
                           B, H, L, dk, dv, int(chunk), _ptr(initial_state), _ptr(x_prev), _ptr(win),
                           _ptr(out), _ptr(final_state), wsp, wsn, _stream(stream))
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
             want_state: bool = True, stream=None, workspace=None):
    """falcon_fwd_host_ws: the forward of one or several variants over the
    same inputs in host memory (CPU tensors; pinned memory lets the library
    overlap the copies of one batch slice with the compute of the next).
    q,k [B,H,L,dk], v [B,H,L,dv], beta [B,H,L] or [B,H,L,dv] (same dtype),
    lam [H] fp32.  The device block (inputs, outputs, the forward's
    workspace) is `workspace` or drawn here from torch's allocator.  Returns
    (outs, states): lists of CPU tensors, one per variant (pinned when
    allocated here).  The call only enqueues; synchronise the stream before
    reading the results."""
    lib = load()
    if isinstance(variants, str):
        variants = [variants]
    n = len(variants)
    if n < 1:
        raise FalconError("at least one variant")
    B, H, L, dk, dv = check_fwd_shapes(variants[0], q, k, v, beta, lam, window)
    for x in variants[1:]:
        check_fwd_shapes(x, q, k, v, beta, lam, window)
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
    for o in out:
        if tuple(o.shape) != (B, H, L, dv) or o.dtype != q.dtype:
            _shape_error("every out must be %s of q's dtype" % ((B, H, L, dv),))
    vids = (ctypes.c_int * n)(*(VARIANTS[x] for x in variants))
    outs = (ctypes.c_void_p * n)(*(_host_ptr(o) for o in out))
    states = None
    if final_state is not None:
        for st in final_state:
            if st is not None and (st.dtype != torch.float32 or tuple(st.shape) != (B, H, dv, dk)):
                _shape_error("final states are fp32 %s" % ((B, H, dv, dk),))
        states = (ctypes.c_void_p * n)(*(_host_ptr(st) for st in final_state))
    need = ctypes.c_size_t(0)
    _check(lib.falcon_fwd_host_workspace_size(n, vids, FORMS[form], DTYPES[q.dtype], PAIRINGS[pairing], PHIS[phi],
                                              int(window), B, H, L, dk, dv, int(chunk),
                                              int(final_state is not None), int(slices), ctypes.byref(need)))
    dev = torch.device("cuda", torch.cuda.current_device()) if stream is None else stream.device
    if workspace is None:
        workspace = _alloc_workspace(need.value, dev, stream)
    wsp = _ptr(workspace) if workspace is not None else None
    wsn = workspace.numel() * workspace.element_size() if workspace is not None else 0
    hp = lambda t: ctypes.c_void_p(_host_ptr(t))  # noqa: E731
    rc = lib.falcon_fwd_host_ws(n, vids, FORMS[form], DTYPES[q.dtype], PAIRINGS[pairing], PHIS[phi],
                                hp(q), hp(k), hp(v), hp(beta), hp(lam), float(eps), int(window),
                                B, H, L, dk, dv, int(chunk), outs, states, int(slices), wsp, wsn, _stream(stream))
    _check(rc)
    return out, final_state


def bwd(variant: str, q, k, v, beta, lam, eps: float, dout, dstate=None, window: int = 1, pairing: str = "prefix",
        phi: str = "l2", stream=None, form: str = "recurrent", chunk: int = 64):
    """falcon_bwd_ws: gradients of a loss with respect to q, k, v, beta and
    lambda of a forward from S_0 = 0, given dout = dL/d(out) (dtype of q) and
    dstate = dL/d(final_state) (fp32, or None).  form="recurrent": every
    variant (window for Falcon-3/3A), d_k = d_v in {32, 64, 128};
    form="chunk": the chunk-parallel backward of Falcon-1/1A, bf16, d = 64,
    chunk 64.  The workspace comes from torch's allocator.  Returns a dict of
    fp32 tensors dq, dk, dv, dbeta, dlambda."""
    lib = load()
    B, H, L, dk, dv = check_fwd_shapes(variant, q, k, v, beta, lam, window, out=dout, final_state=dstate)
    if q.dtype not in DTYPES or not (q.dtype == k.dtype == v.dtype == beta.dtype == dout.dtype):
        raise FalconError("q, k, v, beta, dout must share one dtype, fp32 or bf16")
    if lam.dtype != torch.float32 or (dstate is not None and dstate.dtype != torch.float32):
        raise FalconError("lambda and dstate must be fp32")
    f32 = dict(dtype=torch.float32, device=q.device)
    g = {"dq": torch.empty((B, H, L, dk), **f32), "dk": torch.empty((B, H, L, dk), **f32),
         "dv": torch.empty((B, H, L, dv), **f32), "dbeta": torch.empty(tuple(beta.shape), **f32),
         "dlambda": torch.zeros((H,), **f32)}
    need = ctypes.c_size_t(0)
    _check(lib.falcon_bwd_workspace_size(VARIANTS[variant], FORMS[form], DTYPES[q.dtype], PAIRINGS[pairing],
                                         PHIS[phi], int(window), B, H, L, dk, dv, int(chunk), ctypes.byref(need)))
    ws = _alloc_workspace(need.value, q.device, stream)
    rc = lib.falcon_bwd_ws(VARIANTS[variant], FORMS[form], DTYPES[q.dtype], PAIRINGS[pairing], PHIS[phi],
                           _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(lam), float(eps), int(window), B, H, L, dk, dv,
                           int(chunk), _ptr(dout), _ptr(dstate) if dstate is not None else None,
                           _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dbeta"]), _ptr(g["dlambda"]),
                           _ptr(ws), need.value if ws is not None else 0, _stream(stream))
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
    B, H, L, dk, dv = check_fwd_shapes(variant, q, k, v, beta, lam, window, out, final_state)
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


def check_decode_shapes(variant, q, k, v, beta, lam, window, state, x_prev, win, out=None):
    """Checks the arrays of a decode step against q's [N,H,d_k]: k like q, v
    [N,H,d_v], beta [N,H] or [N,H,d_v], lambda [H], state [N,H,d_v,d_k],
    x_prev [N,H,d_k], win [N,H,window-1,d_k+d_v], out [N,H,d_v]."""
    if variant not in VARIANTS:
        raise FalconError("unknown variant %r" % (variant,))
    if q.dim() != 3:
        _shape_error("q must be [N,H,d_k], got %s" % (tuple(q.shape),))
    N, H, dk = q.shape
    if tuple(k.shape) != (N, H, dk):
        _shape_error("k %s must match q %s" % (tuple(k.shape), tuple(q.shape)))
    if v.dim() != 3 or tuple(v.shape[:2]) != (N, H):
        _shape_error("v must be [N,H,d_v], got %s" % (tuple(v.shape),))
    dv = v.shape[2]
    want = (N, H, dv) if variant in ("F2", "F2A") else (N, H)
    if tuple(beta.shape) != want:
        _shape_error("beta of %s must be %s, got %s" % (variant, want, tuple(beta.shape)))
    if tuple(lam.shape) != (H,):
        _shape_error("lambda must be [H] = (%d,), got %s" % (H, tuple(lam.shape)))
    w = _window(variant, window)
    for t, shape, name in ((state, (N, H, dv, dk), "state"), (x_prev, (N, H, dk), "x_prev"),
                           (win, (N, H, w - 1, dk + dv), "win"), (out, (N, H, dv), "out")):
        if t is not None and tuple(t.shape) != shape:
            _shape_error("%s must be %s, got %s" % (name, shape, tuple(t.shape)))
    if w > 1 and win is None:
        raise FalconError("Falcon-3/3A decode needs the window carry")
    for t in (state, x_prev, win):
        if t is not None and t.dtype != torch.float32:
            raise FalconError("state, x_prev and win are fp32")
    return N, H, dk, dv


def decode_step(variant: str, q, k, v, beta, lam, eps: float, window: int, state, x_prev, win=None,
                out=None, stream=None, pairing: str = "prefix"):
    """falcon_decode_step_ex: q,k [N,H,dk], v [N,H,dv], beta [N,H] or [N,H,dv];
    state [N,H,dv,dk], x_prev [N,H,dk] (may be None under the same-step pair),
    win [N,H,window-1,dk+dv] fp32 (in/out)."""
    lib = load()
    N, H, dk, dv = check_decode_shapes(variant, q, k, v, beta, lam, window, state, x_prev, win, out)
    if x_prev is None and pairing == "prefix":
        raise FalconError("the prefix pair's decode needs x_prev")
    if out is None:
        out = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    rc = lib.falcon_decode_step_ex(VARIANTS[variant], DTYPES[q.dtype], PAIRINGS[pairing], _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(beta), _ptr(lam), float(eps), int(window), N, H, dk, dv, _ptr(state),
                                   _ptr(x_prev), _ptr(win), _ptr(out), _stream(stream))
    _check(rc)
    return out


def carry_from_prefill(variant: str, k, v, window: int, x_prev=None, win=None, stream=None,
                       pairing: str = "prefix"):
    """falcon_decode_carry_from_prefill_ex: returns (x_prev [B,H,dk], win [B,H,w-1,dk+dv])."""
    lib = load()
    if k.dim() != 4 or v.dim() != 4 or tuple(v.shape[:3]) != tuple(k.shape[:3]):
        _shape_error("k [B,H,L,d_k] and v [B,H,L,d_v] must share B,H,L")
    B, H, L, dk = k.shape
    dv = v.shape[-1]
    w = _window(variant, window)
    if x_prev is None:
        x_prev = torch.empty((B, H, dk), dtype=torch.float32, device=k.device)
    if win is None and w > 1:
        win = torch.empty((B, H, w - 1, dk + dv), dtype=torch.float32, device=k.device)
    if tuple(x_prev.shape) != (B, H, dk) or (win is not None and tuple(win.shape) != (B, H, w - 1, dk + dv)):
        _shape_error("x_prev must be [B,H,d_k] and win [B,H,window-1,d_k+d_v]")
    rc = lib.falcon_decode_carry_from_prefill_ex(VARIANTS[variant], DTYPES[k.dtype], PAIRINGS[pairing], _ptr(k),
                                                 _ptr(v), int(window), B, H, L, dk, dv, _ptr(x_prev), _ptr(win),
                                                 _stream(stream))
    _check(rc)
    return x_prev, win
