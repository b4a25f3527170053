"""The caller-owned workspace: falcon_fwd_ws / falcon_bwd_ws give the same
results, bit for bit, as the entry points that draw their workspace from the
device's memory pool, whatever the workspace held before, and they take no
memory from that pool or from torch's allocator."""
import ctypes

import pytest
import torch

from linear_attention_sequence_falcon_b200 import inputs as gen

pytestmark = pytest.mark.gpu

VID = {"F1": 0, "F2": 1, "F3": 2, "F1A": 3, "F2A": 4, "F3A": 5}
FORM = {"recurrent": 0, "masked": 1, "chunk": 2}


@pytest.fixture(scope="module")
def F():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from linear_attention_sequence_falcon_b200 import build
    build.build()
    import linear_attention_sequence_falcon_b200 as F
    F.load()
    return F


def pool_bytes():
    """(reserved, used) bytes of the current device's current memory pool --
    the pool cudaMallocAsync draws from."""
    from cuda.bindings import driver as cu
    cu.cuInit(0)
    err, dev = cu.cuDeviceGet(torch.cuda.current_device())
    assert err == cu.CUresult.CUDA_SUCCESS
    err, pool = cu.cuDeviceGetMemPool(dev)
    assert err == cu.CUresult.CUDA_SUCCESS
    A = cu.CUmemPool_attribute
    err, r = cu.cuMemPoolGetAttribute(pool, A.CU_MEMPOOL_ATTR_RESERVED_MEM_CURRENT)
    err2, u = cu.cuMemPoolGetAttribute(pool, A.CU_MEMPOOL_ATTR_USED_MEM_CURRENT)
    assert err == err2 == cu.CUresult.CUDA_SUCCESS
    return int(r), int(u)


def P(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def allocating_fwd(F, variant, form, d, window, chunk, dev):
    """falcon_fwd_ex: the entry point that draws its own workspace."""
    lib = F.load()
    q, k, v, beta, lam = dev
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    out = torch.empty((B, H, L, dv), dtype=q.dtype, device="cuda")
    S = torch.empty((B, H, dv, dk), dtype=torch.float32, device="cuda")
    rc = lib.falcon_fwd_ex(VID[variant], FORM[form], F.DTYPES[q.dtype], 0, 0, P(q), P(k), P(v), P(beta), P(lam),
                           float(d["eps"]), window, B, H, L, dk, dv, chunk, P(out), P(S),
                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    return out, S


CASES = [("F1", "chunk", "bf16", 2, 3, 300, 64, 64, 1),      # the split tensor-core path (images per chunk)
         ("F1A", "chunk", "bf16", 2, 3, 300, 64, 64, 1),
         ("F2A", "chunk", "bf16", 1, 2, 200, 128, 128, 1),   # per-chunk state images
         ("F3", "masked", "f32", 1, 2, 150, 32, 32, 4),      # masked-parallel unknowns
         ("F1", "masked", "bf16", 1, 2, 130, 64, 64, 1)]


@pytest.mark.parametrize("variant,form,dtype,B,H,L,dk,dv,w", CASES)
def test_caller_workspace_matches_allocating_entry_point(F, variant, form, dtype, B, H, L, dk, dv, w):
    d = gen.draw(variant, B, H, L, dk, dv, seed=700 + L, dtype=dtype)
    dev = [d[n].cuda() for n in ("q", "k", "v", "beta", "lam")]
    need = F.fwd_workspace_size(variant, form, dev[0].dtype, B, H, L, dk, dv, w, 64)
    assert need > 0
    ref_o, ref_S = allocating_fwd(F, variant, form, d, w, 64, dev)
    ws = torch.full((need + 512,), 0xA5, dtype=torch.uint8, device="cuda")  # stale contents must not matter
    for _ in range(2):
        o, S = F.fwd(variant, form, *dev, d["eps"], window=w, chunk=64, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(o, ref_o) and torch.equal(S, ref_S), (variant, form)
        ws.fill_(0x3C)


@pytest.mark.parametrize("variant,form,dtype,B,H,L,dk,dv,w", CASES)
def test_caller_workspace_allocates_nothing(F, variant, form, dtype, B, H, L, dk, dv, w):
    """With the workspace, outputs and state handed in, a call draws nothing
    from the device's memory pool nor from torch's allocator; the allocating
    entry point, for contrast, shows up in the pool while its work is queued."""
    d = gen.draw(variant, B, H, L, dk, dv, seed=710 + L, dtype=dtype)
    dev = [d[n].cuda() for n in ("q", "k", "v", "beta", "lam")]
    need = F.fwd_workspace_size(variant, form, dev[0].dtype, B, H, L, dk, dv, w, 64)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    out = torch.empty((B, H, L, dv), dtype=dev[0].dtype, device="cuda")
    S = torch.empty((B, H, dv, dk), dtype=torch.float32, device="cuda")
    F.fwd(variant, form, *dev, d["eps"], window=w, chunk=64, out=out, final_state=S, workspace=ws)
    torch.cuda.synchronize()
    F.scratch_trim()
    r0, u0 = pool_bytes()
    t0 = torch.cuda.memory_allocated()
    torch.cuda._sleep(50_000_000)  # keep the stream busy so the call's work is still queued below
    F.fwd(variant, form, *dev, d["eps"], window=w, chunk=64, out=out, final_state=S, workspace=ws)
    r1, u1 = pool_bytes()
    assert (r1, u1) == (r0, u0) and torch.cuda.memory_allocated() == t0
    torch.cuda.synchronize()
    assert pool_bytes() == (r0, u0)
    # contrast: the allocating entry point reserves its workspace in the pool
    torch.cuda._sleep(50_000_000)
    allocating_fwd(F, variant, form, d, w, 64, dev)
    r2, _ = pool_bytes()
    torch.cuda.synchronize()
    assert r2 >= r0 + need


def test_backward_workspace_matches_allocating_entry_point(F):
    lib = F.load()
    for variant in ("F1", "F1A"):
        d = gen.draw(variant, 1, 2, 100, 64, 64, seed=720, dtype="f32")
        dev = [d[n].cuda() for n in ("q", "k", "v", "beta", "lam")]
        dout = torch.randn((1, 2, 100, 64), device="cuda")
        g = F.bwd(variant, *dev, d["eps"], dout)
        ref = {n: torch.empty_like(g[n]) for n in g}
        ref["dlambda"].zero_()
        rc = lib.falcon_bwd(VID[variant], 0, 0, 0, *(P(t) for t in dev), float(d["eps"]), 1, 1, 2, 100, 64, 64,
                            P(dout), None, P(ref["dq"]), P(ref["dk"]), P(ref["dv"]), P(ref["dbeta"]),
                            P(ref["dlambda"]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0
        torch.cuda.synchronize()
        for n in g:
            assert torch.equal(g[n], ref[n]), (variant, n)
