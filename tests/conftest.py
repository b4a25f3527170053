import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session", autouse=True)
def no_block_gave_up_in_the_session():
    """After the whole run: no tensor-core thread block gave up on a bounded
    wait.  A block that gives up leaves its outputs incomplete while the call
    still returns FALCON_OK, so every GPU test above counts only if this
    counter stayed at zero (it is read only when the library was loaded on a
    CUDA device during the session)."""
    yield
    try:
        import torch
        if not torch.cuda.is_available():
            return
        from linear_attention_sequence_falcon_b200 import _lib
    except Exception:
        return
    if _lib._lib is None:
        return
    assert _lib.wait_timeouts() == 0, "a tensor-core thread block gave up on a bounded wait during the tests"
