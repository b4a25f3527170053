"""Failure detection on the GPU without a fault: every wait the tensor-core
kernels make on the device is bounded, and a wait that runs out reports
itself and lets the kernel leave (the device stays usable)."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from linear_attention_sequence_falcon_b200 import build
    build.build()
    import linear_attention_sequence_falcon_b200 as F
    F.load()
    return F


def test_bounded_wait_gives_up_and_device_stays_usable(F):
    import time
    t0 = time.time()
    assert F.selftest_bounded_wait(2000) == 1  # a never-completed phase: the wait must give up
    assert time.time() - t0 < 10
    x = torch.arange(1000, device="cuda", dtype=torch.float32)
    assert float(x.sum()) == 499500.0  # the context is intact
    assert F.selftest_bounded_wait(500) == 1


def test_no_kernel_gave_up_during_the_suite(F):
    """The tensor-core kernels count blocks that gave up waiting; a healthy
    run leaves the counter at zero."""
    from linear_attention_sequence_falcon_b200 import inputs as gen
    d = gen.draw("F1", 2, 3, 300, 64, 64, seed=4, dtype="bf16")
    F.fwd("F1", "chunk", *(d[n].cuda() for n in ("q", "k", "v", "beta", "lam")), d["eps"], chunk=64)
    torch.cuda.synchronize()
    assert F.wait_timeouts() == 0
