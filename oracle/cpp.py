"""ctypes binding of the C++ loop oracle (oracle/moe_oracle.cpp).

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` import this module; the product
path never does.

The functions have the names, arguments and results of the NumPy oracle in
oracle/moe_oracle.py, so that every pin runs against both.  The arithmetic is
all in the C++ source; this module only converts arrays and calls it.

The library is compiled from oracle/moe_oracle.cpp with g++ (no CUDA) by
``build()``, and on first use when it is missing or older than its source.
``load(path)`` binds another build of the same source (the mutant tests
compile altered copies).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.cpp")
LIB = os.path.join(HERE, "libmoe_oracle.so")

ACT_RELU, ACT_SWIGLU = 0, 1
GATE_SWITCH, GATE_RENORM = 0, 1
_F64, _F32, _BF16 = 0, 1, 2

_i64, _dbl, _int, _vp = ctypes.c_int64, ctypes.c_double, ctypes.c_int, ctypes.c_void_p


def compile_library(src: str = SRC, out: str = LIB, opt: str = "-O3") -> str:
    """g++ -shared build of the oracle source (plain C++17, pthreads)."""
    cmd = ["g++", opt, "-std=c++17", "-shared", "-fPIC", "-pthread", src, "-o", out]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"g++ failed on {src}:\n{r.stdout}\n{r.stderr}")
    return out


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        compile_library()
    return LIB


def _widen(a: np.ndarray, code: int) -> np.ndarray:
    """float64 copy of a host array returned by _float_array."""
    if code == _BF16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


class _Result(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("logits", "p", "lse", "idx", "gate", "counts", "kept_counts", "offsets",
                                   "rank", "kept", "dest_row")] + [
        ("dropped", _i64), ("capacity", _i64), ("aux", _dbl), ("z", _dbl), ("balance", _dbl * 3), ("y", _vp)]


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else _vp(a.ctypes.data)


def _float_array(a):
    """(contiguous host array, type code) of a float tensor: numpy float64 /
    float32, or a torch tensor (bf16 kept as its bit patterns); per-expert
    sequences (lists, lazily converted host copies) are stacked."""
    if a is None:
        return None, _F64
    try:
        import torch
        if isinstance(a, torch.Tensor):
            t = a.detach().cpu().contiguous()
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy().view(np.uint16), _BF16
            if t.dtype == torch.float32:
                return t.numpy(), _F32
            return t.double().numpy(), _F64
    except ImportError:
        pass
    if not isinstance(a, np.ndarray):
        if hasattr(a, "__len__") and hasattr(a, "__getitem__"):
            a = np.stack([np.asarray(a[i]) for i in range(len(a))])
        else:
            a = np.asarray(a)
    if a.dtype == np.float32:
        return np.ascontiguousarray(a), _F32
    return np.ascontiguousarray(a, dtype=np.float64), _F64


class Oracle:
    """The C++ oracle bound to one build of its library."""

    ACT_RELU, ACT_SWIGLU = ACT_RELU, ACT_SWIGLU
    GATE_SWITCH, GATE_RENORM = GATE_SWITCH, GATE_RENORM

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        lib.orc_router_logits.argtypes = [_i64, _i64, _i64, _vp, _int, _vp, _int, _vp, _int, _int, _vp]
        lib.orc_softmax_lse.argtypes = [_i64, _i64, _vp, _vp, _vp]
        lib.orc_top_k.argtypes = [_i64, _i64, _i64, _vp, _vp]
        lib.orc_gates.argtypes = [_i64, _i64, _i64, _vp, _vp, _vp, _int, _vp]
        lib.orc_expert_capacity.argtypes = [_dbl, _i64, _i64, _i64]
        lib.orc_expert_capacity.restype = _i64
        lib.orc_assign_slots.argtypes = [_i64, _i64, _i64, _vp, _i64] + [_vp] * 7
        lib.orc_expert_ffn.argtypes = [_i64, _i64, _i64, _int, _vp, _vp, _vp, _vp, _int, _vp, _int]
        lib.orc_aux_and_z.argtypes = [_i64, _i64, _i64, _vp, _vp, _vp, _vp]
        lib.orc_balance_losses.argtypes = [_i64, _i64, _i64, _vp, _vp, _vp]
        lib.orc_moe_forward.argtypes = ([_i64, _i64, _i64, _i64, _i64, _int, _int, _dbl, _vp, _int, _vp, _int,
                                         _vp, _int, _vp, _int, _vp, _vp, _vp, _int, _i64, _vp, _vp, _vp, _vp,
                                         _i64, _int, ctypes.POINTER(_Result)])
        lib.orc_moe_forward.restype = _int
        lib.orc_hardware_threads.restype = _int
        self.lib = lib
        self.path = path

    def hardware_threads(self) -> int:
        return int(self.lib.orc_hardware_threads())

    # --------------------------------------------------------------- steps
    def router_logits(self, x, W_r, b_r=None, dtype=np.float32) -> np.ndarray:
        X, xt = _float_array(x)
        W, wt = _float_array(W_r)
        B, bt = _float_array(b_r)
        T, d = X.shape
        E = W.shape[0]
        h = np.empty((T, E), np.float64)
        self.lib.orc_router_logits(T, d, E, _ptr(X), xt, _ptr(W), wt, _ptr(B), bt,
                                   1 if dtype == np.float32 else 0, _ptr(h))
        return h.astype(dtype)

    def softmax_lse(self, h32):
        h = np.ascontiguousarray(h32, np.float64)
        T, E = h.shape
        p = np.empty((T, E), np.float64)
        lse = np.empty(T, np.float64)
        self.lib.orc_softmax_lse(T, E, _ptr(h), _ptr(p), _ptr(lse))
        return p, lse

    def top_k(self, h32, k: int) -> np.ndarray:
        h = np.ascontiguousarray(h32, np.float64)
        T, E = h.shape
        idx = np.empty((T, k), np.int64)
        self.lib.orc_top_k(T, E, k, _ptr(h), _ptr(idx))
        return idx

    def gates(self, h32, p, idx, gate_mode: int) -> np.ndarray:
        h = np.ascontiguousarray(h32, np.float64)
        p = np.ascontiguousarray(p, np.float64)
        idx = np.ascontiguousarray(idx, np.int64)
        T, k = idx.shape
        g = np.empty((T, k), np.float64)
        self.lib.orc_gates(T, h.shape[1] if h.ndim == 2 else 0, k, _ptr(h), _ptr(p), _ptr(idx), int(gate_mode),
                           _ptr(g))
        return g

    def expert_capacity(self, capacity_factor: float, T: int, k: int, E: int) -> Optional[int]:
        c = int(self.lib.orc_expert_capacity(float(capacity_factor), T, k, E))
        return None if c < 0 else c

    def assign_slots(self, idx, E: int, C: Optional[int]) -> dict:
        idx = np.ascontiguousarray(idx, np.int64)
        T, k = idx.shape
        counts = np.empty(E, np.int64)
        kept_counts = np.empty(E, np.int64)
        offsets = np.empty(E + 1, np.int64)
        rank = np.empty((T, k), np.int64)
        kept = np.empty((T, k), np.uint8)
        dest = np.empty((T, k), np.int64)
        dropped = np.zeros(1, np.int64)
        self.lib.orc_assign_slots(T, k, E, _ptr(idx), -1 if C is None else int(C), _ptr(counts), _ptr(kept_counts),
                                  _ptr(offsets), _ptr(rank), _ptr(kept), _ptr(dest), _ptr(dropped))
        return {"counts": counts, "kept_counts": kept_counts, "offsets": offsets, "rank": rank,
                "kept": kept.astype(bool), "dest_row": dest, "dropped": int(dropped[0])}

    def expert_ffn(self, xr, W1e, W3e, W2e, act: int, threads: int = 1) -> np.ndarray:
        x = np.ascontiguousarray(xr, np.float64)
        W1, t1 = _float_array(W1e)
        W2, t2 = _float_array(W2e)
        W3, t3 = _float_array(W3e)
        if t2 != t1 or (W3 is not None and t3 != t1):  # one element type for the three
            W1, W2, t1 = _float_array(_widen(W1, t1))[0], _float_array(_widen(W2, t2))[0], _F64
            W3 = None if W3 is None else _float_array(_widen(W3, t3))[0]
        n, d = x.shape
        d_ff = W1.shape[0]
        out = np.empty((n, d), np.float64)
        self.lib.orc_expert_ffn(n, d, d_ff, int(act), _ptr(x), _ptr(W1), _ptr(W3), _ptr(W2), t1, _ptr(out), threads)
        return out

    def aux_and_z(self, p, lse, idx, E: int):
        p = np.ascontiguousarray(p, np.float64)
        lse = np.ascontiguousarray(lse, np.float64)
        idx = np.ascontiguousarray(idx, np.int64)
        T, k = idx.shape
        out = np.zeros(2, np.float64)
        self.lib.orc_aux_and_z(T, E, k, _ptr(p), _ptr(lse), _ptr(idx), _ptr(out))
        return float(out[0]), float(out[1])

    def balance_losses(self, p, idx, E: int) -> dict:
        p = np.ascontiguousarray(p, np.float64)
        idx = np.ascontiguousarray(idx, np.int64)
        T, k = idx.shape
        out = np.zeros(3, np.float64)
        self.lib.orc_balance_losses(T, E, k, _ptr(p), _ptr(idx), _ptr(out))
        return {"aux_all_choices": float(out[0]), "cv_counts": float(out[1]), "cv2_probs": float(out[2])}

    # --------------------------------------------------------------- whole layer
    def moe_forward(self, x, W_r, b_r, W1, W3, W2, *, k: int, gate_mode: int, act: int, capacity_factor: float,
                    rows: Optional[Sequence[int]] = None, logits: Optional[np.ndarray] = None,
                    shared: Optional[tuple] = None, logits_dtype=np.float32, threads: int = 0) -> dict:
        """Same arguments and results as oracle.moe_oracle.moe_forward (see there),
        plus ``threads`` (0: one per hardware thread; the results do not depend on it)."""
        X, xt = _float_array(x)
        WR, wrt = _float_array(W_r)
        BR, brt = _float_array(b_r)
        V1, wt = _float_array(W1)
        V2, wt2 = _float_array(W2)
        V3 = None if W3 is None else _float_array(W3)[0]
        if wt2 != wt or (V3 is not None and V3.dtype != V1.dtype):
            raise ValueError("W1, W3 and W2 must share one dtype")
        T, d = X.shape
        E = WR.shape[0]
        d_ff = V1.shape[-2]
        # the routed experts are the first E of W1 / W3 / W2 (more may follow)
        V1, V2 = V1[:E], V2[:E]
        V3 = None if V3 is None else V3[:E]
        ns, S1, S3, S2 = 0, None, None, None
        if shared is not None:
            ns = len(shared[0])
            S1 = _float_array(shared[0])[0]
            S3 = None if shared[1] is None else _float_array(shared[1])[0]
            S2 = _float_array(shared[2])[0]
            for s in (S1, S2) + (() if S3 is None else (S3,)):
                if s.dtype != V1.dtype:
                    raise ValueError("shared experts must have the routed experts' dtype")
        V1, V2 = np.ascontiguousarray(V1), np.ascontiguousarray(V2)
        V3 = None if V3 is None else np.ascontiguousarray(V3)
        LG = None if logits is None else np.ascontiguousarray(logits, np.float64)
        want = np.arange(T, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, np.int64)
        res = {
            "logits": np.empty((T, E), np.float64), "p": np.empty((T, E), np.float64), "lse": np.empty(T),
            "idx": np.empty((T, k), np.int64), "gate": np.empty((T, k), np.float64),
            "counts": np.empty(E, np.int64), "kept_counts": np.empty(E, np.int64),
            "offsets": np.empty(E + 1, np.int64), "rank": np.empty((T, k), np.int64),
            "kept": np.empty((T, k), np.uint8), "dest_row": np.empty((T, k), np.int64),
            "y": np.empty((len(want), d), np.float64),
        }
        r = _Result()
        for name in ("logits", "p", "lse", "idx", "gate", "counts", "kept_counts", "offsets", "rank", "kept",
                     "dest_row", "y"):
            setattr(r, name, res[name].ctypes.data)
        rc = self.lib.orc_moe_forward(
            T, d, E, k, d_ff, int(act), int(gate_mode), float(capacity_factor), _ptr(X), xt, _ptr(WR), wrt,
            _ptr(BR), brt, _ptr(LG), 1 if logits_dtype == np.float32 else 0, _ptr(V1), _ptr(V3), _ptr(V2), wt, ns,
            _ptr(S1), _ptr(S3), _ptr(S2), None if rows is None else _ptr(want), len(want), int(threads),
            ctypes.byref(r))
        if rc != 0:
            raise ValueError("orc_moe_forward: bad sizes")
        res["logits"] = res["logits"].astype(logits_dtype)
        res["kept"] = res["kept"].astype(bool)
        res.update(dropped=int(r.dropped), capacity=None if r.capacity < 0 else int(r.capacity), aux=float(r.aux),
                   z=float(r.z), rows=want, aux_all_choices=float(r.balance[0]), cv_counts=float(r.balance[1]),
                   cv2_probs=float(r.balance[2]))
        return res


_DEFAULT: Optional[Oracle] = None


def load(path: Optional[str] = None) -> Oracle:
    """The oracle bound to ``path`` (default: the library built from oracle/moe_oracle.cpp)."""
    global _DEFAULT
    if path is not None:
        return Oracle(path)
    if _DEFAULT is None:
        _DEFAULT = Oracle(build())
    return _DEFAULT
