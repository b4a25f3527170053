"""Falcon fast-weight updates (Fast Weight Attention) on B200 (sm_100a).

The computation lives in libfalcon.so (C ABI in include/falcon.h, CUDA
kernels in csrc/); this package is the thin ctypes binding plus the seeded
synthetic-input generator.
"""
from ._lib import (DTYPES, EXPORTS, FORMS, LIB_PATH, VARIANTS, FalconError, carry_from_prefill,  # noqa: F401
                   bwd, check_decode_shapes, check_fwd_shapes, decode_step, fwd, fwd_host, fwd_masked_noalloc,
                   fwd_workspace_size, load, scratch_trim, selftest_bounded_wait, wait_timeouts)
