"""Sparse Mixture-of-Experts layer forward pass for B200 (sm_100a).

The layer is computed by the CUDA library ``libmoe_b200.so`` (C ABI in
include/moe.h); this package is its thin Python binding plus the seeded
synthetic workloads used by the tests and the benchmark.
"""
from .layer import MoELayer, clear_status, launch_count, quantize_int4, selftest_timeout, status  # noqa: F401
from ._lib import LIB_PATH, MoEError  # noqa: F401
