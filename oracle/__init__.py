"""fp64 CPU oracle for the Falcon fast-weight updates -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (the CUDA library and its
binding) never does, and this package never imports the product: the two
share no code.  Seeded inputs come from a separate generator module that holds
none of the method's arithmetic.

``falcon_oracle.c`` is the plain fp64 statement of the method (recurrent
definition, masked-parallel and chunk-parallel unrollings, the decode step,
and the reverse mode of the recurrent definition for the backward pass);
``brute.py`` is an independent numpy re-derivation (products of transition
matrices) for tiny sizes.  Both cite the pages by title and section:
  [EXPL] "Fast Weight Attention：用于持续学习的快速权重注意力", 核心方法
  [SUMM] "Fast Weight Attention for Continual Learning", 方法
  [NEWS] "借鉴40年前的设想！字节Seed提出快速权重注意力推进大模型持续学习", 02
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "falcon_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

VARIANTS = {"F1": 0, "F2": 1, "F3": 2, "F1A": 3, "F2A": 4, "F3A": 5}
FORMS = {"recurrent": 0, "masked": 1, "chunk": 2}
PAIRINGS = {"prefix": 0, "same_step": 1}
PHIS = {"l2": 0, "identity": 1}

_lib = None


def build(force: bool = False) -> str:
    """Compile falcon_oracle.c with gcc into liboracle.so (in-tree)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC,
                               "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        I, D = ctypes.c_int, ctypes.c_double
        lib.oracle_fwd.argtypes = [I, I, I, I, dp, dp, dp, dp, dp, D, I, I, I, I, I, I, I, dp, dp, I]
        lib.oracle_fwd.restype = I
        lib.oracle_decode_step.argtypes = [I, I, I, dp, dp, dp, dp, dp, D, I, I, I, I, I, dp, dp, dp, dp]
        lib.oracle_decode_step.restype = I
        lib.oracle_carry_from_prefill.argtypes = [I, I, I, dp, dp, I, I, I, I, I, I, dp, dp]
        lib.oracle_carry_from_prefill.restype = I
        lib.oracle_fwd_carry.argtypes = [I, I, I, dp, dp, dp, dp, dp, D, I, I, I, I, I, I, dp, dp, dp, dp, dp, I]
        lib.oracle_fwd_carry.restype = I
        lib.oracle_bwd.argtypes = [I, I, I, dp, dp, dp, dp, dp, D, I, I, I, I, I, I, dp, dp, dp, dp, dp, dp, dp, I, dp]
        lib.oracle_bwd.restype = I
        _lib = lib
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def per_channel(variant: str) -> bool:
    return variant in ("F2", "F2A")


def fwd(variant, form, q, k, v, beta, lam, eps, window=1, chunk=64,
        pairing="prefix", phi="l2", nthreads=0, return_threads=False):
    """Run the oracle on fp64 arrays q,k [B,H,L,dk], v [B,H,L,dv],
    beta [B,H,L] or [B,H,L,dv], lam [H].  Returns (out [B,H,L,dv], S_L [B,H,dv,dk])."""
    lib = _load()
    q, k, v, beta, lam = map(_f64, (q, k, v, beta, lam))
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, H, L, dv))
    fs = np.zeros((B, H, dv, dk))
    rc = lib.oracle_fwd(VARIANTS[variant], FORMS[form], PAIRINGS[pairing], PHIS[phi],
                        _p(q), _p(k), _p(v), _p(beta), _p(lam), float(eps), int(window),
                        B, H, L, dk, dv, int(chunk), _p(out), _p(fs), int(nthreads))
    if rc < 0:
        raise ValueError("oracle_fwd rejected its arguments (code %d)" % rc)
    if return_threads:
        return out, fs, rc
    return out, fs


def decode_step(variant, q, k, v, beta, lam, eps, window, state, x_prev, win, phi="l2", pairing="prefix"):
    """One decode step on fp64 arrays; state, x_prev and win are updated in
    place (x_prev may be None under the same-step pair)."""
    lib = _load()
    q, k, v, beta, lam = map(_f64, (q, k, v, beta, lam))
    for a in (state, x_prev, win):
        assert a is None or (a.dtype == np.float64 and a.flags.c_contiguous)
    N, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((N, H, dv))
    null = ctypes.POINTER(ctypes.c_double)()
    rc = lib.oracle_decode_step(VARIANTS[variant], PAIRINGS[pairing], PHIS[phi], _p(q), _p(k), _p(v), _p(beta),
                                _p(lam), float(eps), int(window), N, H, dk, dv,
                                _p(state), _p(x_prev) if x_prev is not None else null, _p(win), _p(out))
    if rc < 0:
        raise ValueError("oracle_decode_step rejected its arguments (code %d)" % rc)
    return out


def carry_from_prefill(variant, k, v, window, phi="l2", pairing="prefix"):
    """Decode carry (x_prev [B,H,dk], win [B,H,max(Bw-1,0),dk+dv]) after a prefill."""
    lib = _load()
    k, v = _f64(k), _f64(v)
    B, H, L, dk = k.shape
    dv = v.shape[-1]
    w = window if variant in ("F3", "F3A") else 1
    x_prev = np.zeros((B, H, dk))
    win = np.zeros((B, H, max(w - 1, 0), dk + dv))
    rc = lib.oracle_carry_from_prefill(VARIANTS[variant], PAIRINGS[pairing], PHIS[phi], _p(k), _p(v), int(window),
                                       B, H, L, dk, dv, _p(x_prev), _p(win))
    if rc < 0:
        raise ValueError("oracle_carry_from_prefill rejected its arguments (code %d)" % rc)
    return x_prev, win


def fwd_carry(variant, q, k, v, beta, lam, eps, window=1, S0=None, x_prev=None, win=None, phi="l2",
              nthreads=0, pairing="prefix"):
    """Recurrent definition over a segment that continues a sequence: state
    S0 [B,H,dv,dk] and the decode carry x_prev [B,H,dk], win [B,H,Bw-1,dk+dv]
    (each None = zeros, the start of a sequence; x_prev is not read under the
    same-step pair).  Returns (out [B,H,L,dv], S_L [B,H,dv,dk])."""
    lib = _load()
    q, k, v, beta, lam = map(_f64, (q, k, v, beta, lam))
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    null = ctypes.POINTER(ctypes.c_double)()
    carry = [_f64(a) if a is not None else None for a in (S0, x_prev, win)]
    if carry[2] is not None and carry[2].size == 0:
        carry[2] = None
    ptrs = [_p(a) if a is not None else null for a in carry]
    out = np.zeros((B, H, L, dv))
    fs = np.zeros((B, H, dv, dk))
    rc = lib.oracle_fwd_carry(VARIANTS[variant], PAIRINGS[pairing], PHIS[phi], _p(q), _p(k), _p(v), _p(beta), _p(lam),
                              float(eps), int(window), B, H, L, dk, dv, *ptrs, _p(out), _p(fs), int(nthreads))
    if rc < 0:
        raise ValueError("oracle_fwd_carry rejected its arguments (code %d)" % rc)
    return out, fs


def bwd(variant, q, k, v, beta, lam, eps, dout, dstate=None, window=1, pairing="prefix", phi="l2", nthreads=0):
    """Reverse mode of the recurrent definition (S_0 = 0): given dL/dout
    [B,H,L,dv] and dL/dS_L [B,H,dv,dk] (None: zero), returns dq, dk, dv
    (shapes of q, k, v), dbeta (shape of beta), dlambda [H] and
    dlambda_l1 [H], the sum of the magnitudes of the terms dlambda adds up."""
    lib = _load()
    q, k, v, beta, lam, dout = map(_f64, (q, k, v, beta, lam, dout))
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    dq, dkk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dbeta, dlam, dlam_l1 = np.zeros_like(beta), np.zeros(H), np.zeros(H)
    ds = None if dstate is None else _f64(dstate)
    rc = lib.oracle_bwd(VARIANTS[variant], PAIRINGS[pairing], PHIS[phi], _p(q), _p(k), _p(v), _p(beta), _p(lam),
                        float(eps), int(window), B, H, L, dk, dv, _p(dout), None if ds is None else _p(ds),
                        _p(dq), _p(dkk), _p(dvv), _p(dbeta), _p(dlam), int(nthreads), _p(dlam_l1))
    if rc < 0:
        raise ValueError("oracle_bwd rejected its arguments (code %d)" % rc)
    return {"dq": dq, "dk": dkk, "dv": dvv, "dbeta": dbeta, "dlambda": dlam, "dlambda_l1": dlam_l1}
