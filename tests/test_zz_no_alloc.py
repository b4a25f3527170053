"""falcon_fwd_masked_noalloc against falcon_fwd's masked form.

The allocation-free entry point serves callers that may not allocate device
memory (a host that owns every device allocation and gives the library only
its input and output buffers, or a service with a fixed memory budget).  It
must give the same results as the allocating entry point, call after call,
although every call reuses the same fixed scratch array inside the library.
This file is collected last so that a run stopping at its first failure has
already run every other test; it also passes when run alone.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_sequence_falcon_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def pool_bytes():
    """(reserved, used) bytes of the current device's current memory pool."""
    from cuda.bindings import driver as cu
    cu.cuInit(0)
    _, dev = cu.cuDeviceGet(torch.cuda.current_device())
    _, pool = cu.cuDeviceGetMemPool(dev)
    A = cu.CUmemPool_attribute
    _, r = cu.cuMemPoolGetAttribute(pool, A.CU_MEMPOOL_ATTR_RESERVED_MEM_CURRENT)
    _, u = cu.cuMemPoolGetAttribute(pool, A.CU_MEMPOOL_ATTR_USED_MEM_CURRENT)
    return int(r), int(u)


@pytest.fixture(scope="module")
def F():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from linear_attention_sequence_falcon_b200 import build
    build.build()
    import linear_attention_sequence_falcon_b200 as F
    F.load()
    return F


def rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


def _pair(F, variant, dtype, B, H, L, dk, dv, seed, window):
    """The same kernel on the same inputs as falcon_fwd's masked form: the
    results must be identical bit for bit (a scratch mix-up would show), and
    within the parity tolerance of the fp64 oracle."""
    d = gen.draw(variant, B, H, L, dk, dv, seed=seed, dtype=dtype)
    args = [d[n].cuda() for n in ("q", "k", "v", "beta", "lam")]
    ref_o, ref_S = F.fwd(variant, "masked", *args, d["eps"], window=window)
    o, S = F.fwd_masked_noalloc(variant, *args, d["eps"], window=window)
    torch.cuda.synchronize()
    assert torch.equal(o, ref_o) and torch.equal(S, ref_S), (variant, dtype)
    oo, oS = oracle.fwd(variant, "recurrent", d["q_64"], d["k_64"], d["v_64"], d["beta_64"], d["lam_64"],
                        d["eps_64"], window=window)
    tol = TOL[dtype]
    assert rel(o, torch.from_numpy(oo)) <= tol and rel(S, torch.from_numpy(oS)) <= tol, (variant, dtype)
    return o, S


def test_noalloc_matches_allocating_entry_point_twice(F):
    """Two calls in a row (different variants, dtypes and shapes, so the
    second call sees the first one's leftovers in the shared scratch)."""
    _pair(F, "F3", "f32", 2, 3, 300, 64, 64, seed=11, window=4)
    _pair(F, "F1", "bf16", 3, 2, 257, 128, 64, seed=12, window=1)


def test_noalloc_repeat_same_inputs(F):
    """The same inputs twice give the same answer both times."""
    o1, S1 = _pair(F, "F2", "bf16", 2, 2, 200, 32, 32, seed=13, window=1)
    o2, S2 = _pair(F, "F2", "bf16", 2, 2, 200, 32, 32, seed=13, window=1)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_noalloc_takes_no_memory(F):
    """On a shape not used before, the call draws nothing from the device's
    memory pool nor from torch's allocator (outputs handed in)."""
    d = gen.draw("F3A", 1, 3, 177, 64, 32, seed=14, dtype="bf16")
    args = [d[n].cuda() for n in ("q", "k", "v", "beta", "lam")]
    out = torch.empty((1, 3, 177, 32), dtype=torch.bfloat16, device="cuda")
    S = torch.empty((1, 3, 32, 64), dtype=torch.float32, device="cuda")
    F.fwd_masked_noalloc("F3A", *args, d["eps"], window=3, out=out, final_state=S)  # set-up call
    torch.cuda.synchronize()
    F.scratch_trim()
    before = pool_bytes(), torch.cuda.memory_allocated()
    torch.cuda._sleep(50_000_000)
    F.fwd_masked_noalloc("F3A", *args, d["eps"], window=3, out=out, final_state=S)
    assert (pool_bytes(), torch.cuda.memory_allocated()) == before
    torch.cuda.synchronize()
    assert (pool_bytes(), torch.cuda.memory_allocated()) == before


def test_noalloc_rejects_oversize(F):
    """A problem beyond the fixed scratch is refused with its own status and
    nothing is enqueued."""
    q = torch.zeros((64, 16, 1024, 128), device="cuda", dtype=torch.bfloat16)
    b = torch.zeros((64, 16, 1024), device="cuda", dtype=torch.bfloat16)
    lam = torch.zeros(16, device="cuda")
    with pytest.raises(F.FalconError, match="-10"):
        F.fwd_masked_noalloc("F1", q, q, q, b, lam, 1e-6)
