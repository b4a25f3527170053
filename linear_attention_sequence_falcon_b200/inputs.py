"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and rounds them to the kernel's input dtype;
it holds none of the Falcon arithmetic.  Both the CUDA path and the fp64
oracle consume what it returns: the GPU gets the dtype-rounded tensors, the
oracle gets the very same rounded values upcast to fp64, so a parity gap
measures kernel error only.

Workloads stand in for the ~124M-parameter language models the pages train
(12 heads of 64 channels, sequences of 2K and longer); q, k, v ~ N(0,1),
beta = sigmoid(N(0,1)), lambda ~ U(0, 0.05) per head unless fixed, eps = 1e-6.
Random streams: numpy PCG64 seeded per workload.
"""
from __future__ import annotations

import numpy as np
import torch

PER_CHANNEL_BETA = ("F2", "F2A")


def _round(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def draw(variant: str, B: int, H: int, L: int, dk: int, dv: int, seed: int,
         lam=None, dtype: str = "bf16", eps: float = 1e-6, key_scale: float = 1.0):
    """Draw one forward workload.

    lam: None -> U(0, 0.05) per head; a float -> that value for every head;
    an array -> used as given.  Returns a dict of CPU torch tensors in the
    kernel dtype (q, k, v, beta; lam and eps as fp32) plus fp64 numpy copies
    of the identical values under the suffix ``_64``.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    q = rng.standard_normal((B, H, L, dk), dtype=np.float32)
    k = rng.standard_normal((B, H, L, dk), dtype=np.float32) * np.float32(key_scale)
    v = rng.standard_normal((B, H, L, dv), dtype=np.float32)
    bshape = (B, H, L, dv) if variant in PER_CHANNEL_BETA else (B, H, L)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(bshape, dtype=np.float32)))
    if lam is None:
        lam_a = rng.uniform(0.0, 0.05, size=H).astype(np.float32)
    elif np.isscalar(lam):
        lam_a = np.full(H, lam, dtype=np.float32)
    else:
        lam_a = np.asarray(lam, dtype=np.float32)
    d = {
        "q": _round(q, dtype), "k": _round(k, dtype), "v": _round(v, dtype),
        "beta": _round(beta.astype(np.float32), dtype),
        "lam": torch.from_numpy(lam_a.copy()),
        "eps": float(np.float32(eps)),
    }
    for name in ("q", "k", "v", "beta"):
        d[name + "_64"] = d[name].to(torch.float64).numpy()
    d["lam_64"] = lam_a.astype(np.float64)
    d["eps_64"] = float(np.float32(eps))
    d["shape"] = dict(B=B, H=H, L=L, dk=dk, dv=dv)
    d["variant"] = variant
    d["dtype"] = dtype
    return d


def draw_decode(variant: str, N: int, H: int, dk: int, dv: int, steps: int, seed: int,
                lam=0.02, dtype: str = "bf16", eps: float = 1e-6):
    """Per-step decode inputs: q,k [steps,N,H,dk], v [steps,N,H,dv],
    beta [steps,N,H] or [steps,N,H,dv]; same conventions as ``draw``."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = rng.standard_normal((steps, N, H, dk), dtype=np.float32)
    k = rng.standard_normal((steps, N, H, dk), dtype=np.float32)
    v = rng.standard_normal((steps, N, H, dv), dtype=np.float32)
    bshape = (steps, N, H, dv) if variant in PER_CHANNEL_BETA else (steps, N, H)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(bshape, dtype=np.float32)))
    lam_a = (rng.uniform(0.0, 0.05, size=H) if lam is None else np.full(H, lam)).astype(np.float32)
    d = {
        "q": _round(q, dtype), "k": _round(k, dtype), "v": _round(v, dtype),
        "beta": _round(beta.astype(np.float32), dtype),
        "lam": torch.from_numpy(lam_a.copy()), "eps": float(np.float32(eps)),
    }
    for name in ("q", "k", "v", "beta"):
        d[name + "_64"] = d[name].to(torch.float64).numpy()
    d["lam_64"] = lam_a.astype(np.float64)
    d["eps_64"] = float(np.float32(eps))
    return d


# The five workloads (shapes and hyper-parameters as the benchmark spec fixes
# them); seed = 20260000 + workload number.
WORKLOADS = {
    1: dict(name="falcon1-recurrent-fp32-1x1x64x16", variants=("F1",), forms=("recurrent",),
            B=1, H=1, L=64, dk=16, dv=16, chunk=64, window=1, lam=0.01, dtype="f32"),
    2: dict(name="falcon1-1A-chunk-bf16-8x12x2048x64", variants=("F1", "F1A"), forms=("chunk",),
            B=8, H=12, L=2048, dk=64, dv=64, chunk=64, window=1, lam=None, dtype="bf16"),
    3: dict(name="falcon2-chunk-bf16-4x16x4096x128", variants=("F2",), forms=("chunk",),
            B=4, H=16, L=4096, dk=128, dv=128, chunk=64, window=1, lam=None, dtype="bf16"),
    4: dict(name="falcon3-3A-window4-bf16-8x12x2048x64", variants=("F3", "F3A"),
            forms=("masked", "chunk"), B=8, H=12, L=2048, dk=64, dv=64, chunk=64, window=4,
            lam=None, dtype="bf16"),
    5: dict(name="falcon2A-prefill-bf16-2x16x32768x128", variants=("F2A",), forms=("chunk",),
            B=2, H=16, L=32768, dk=128, dv=128, chunk=64, window=1, lam=0.02, dtype="bf16",
            decode=dict(N=64, H=16, dk=128, dv=128, steps=4096)),
}


def workload_inputs(n: int, variant: str, **override):
    w = dict(WORKLOADS[n])
    w.update(override)
    return draw(variant, w["B"], w["H"], w["L"], w["dk"], w["dv"], seed=20260000 + n,
                lam=w["lam"], dtype=w["dtype"])
