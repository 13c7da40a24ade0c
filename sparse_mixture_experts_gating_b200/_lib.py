"""ctypes view of libmoe_b200.so (the C ABI declared in include/moe.h).

Argument marshalling only.  Loading fails loudly when the library has not
been built: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_float, c_int, c_int64, c_size_t, c_uint64, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_RANGE = 0, 1, 2, 3, 4, 5
STAGES = ("router", "scan", "dispatch", "gemm1", "gemm2", "combine")

# Every entry point of include/moe.h, with its ctypes signature.
SIGNATURES = {
    "moe_create": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int, c_double, c_int, POINTER(c_void_p)]),
    "moe_set_hidden_precision": (c_int, [c_void_p, c_int]),
    "moe_destroy": (c_int, [c_void_p]),
    "moe_capacity": (c_int64, [c_void_p, c_int64]),
    "moe_workspace_bytes": (c_size_t, [c_void_p, c_int64]),
    "moe_set_shared_experts": (c_int, [c_void_p, c_int]),
    "moe_balance_losses": (c_int, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p]),
    "moe_forward": (c_int, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                            c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p,
                            c_void_p]),
    "moe_forward_static": (c_int, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                   c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "moe_backward_workspace_bytes": (c_size_t, [c_void_p, c_int64]),
    "moe_backward": (c_int, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                             c_void_p, c_float, c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                             c_void_p, c_void_p, c_size_t, c_void_p, c_size_t, c_void_p]),
    "moe_quantize_int4": (c_int, [c_void_p, c_int64, c_int64, c_void_p, c_void_p, c_void_p]),
    "moe_workspace_bytes_w4": (c_size_t, [c_void_p, c_int64]),
    "moe_forward_w4": (c_int, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                               c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                               c_void_p, c_size_t, c_void_p, c_void_p]),
    "moe_status": (c_int, [c_void_p]),
    "moe_clear_status": (c_int, []),
    "moe_last_error": (c_char_p, []),
    "moe_launch_count": (c_uint64, []),
    "moe_selftest_timeout": (c_int, [c_int64, c_void_p]),
}


class MoEDebug(ctypes.Structure):
    _fields_ = [
        ("logits_in", c_void_p),
        ("logits_out", c_void_p),
        ("lse_out", c_void_p),
        ("topk_idx", c_void_p),
        ("topk_gate", c_void_p),
        ("dest_row", c_void_p),
        ("drop_mask", c_void_p),
        ("expert_offsets", c_void_p),
        ("y_f32", c_void_p),
        ("events", c_void_p * (2 * len(STAGES))),
    ]


class MoEError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[moe error {code}] {msg}")
        self.code = code


_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library (built in-tree by the package's _build module)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m sparse_mixture_experts_gating_b200._build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def check(code: int) -> None:
    if code != MOE_OK:
        raise MoEError(code, lib().moe_last_error().decode())
