"""Python binding of the MoE layer forward pass (torch tensors -> C ABI).

Marshalling only: every step of the layer runs in the CUDA library.  PyTorch
provides device memory and the current stream.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib
from ._lib import MoEDebug, check, lib

ACT = {"relu": 0, "swiglu": 1}
GATE = {"switch": 0, "renorm": 1}
DTYPE = {torch.float32: 0, torch.bfloat16: 1}
HIDDEN = {"bf16x2": 0, "bf16": 1, "f16": 2, "auto": 3}


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _debug_struct(debug: Optional[dict], events, stream) -> Optional[MoEDebug]:
    """moe_debug of the given device tensors and stage events (None if neither)."""
    if debug is None and events is None:
        return None
    dbg = MoEDebug()
    for name, t in (debug or {}).items():
        setattr(dbg, name, _ptr(t))
    if events is not None:
        for i, ev in enumerate(events):
            if ev is not None:
                if not ev.cuda_event:  # torch creates its CUDA event lazily, on first record
                    ev.record(torch.cuda.current_stream() if stream is None else stream)
                dbg.events[i] = ev.cuda_event
    return dbg


class MoELayer:
    """One MoE layer description (E experts, top-k, d -> d_ff -> d experts).

    act: "relu" | "swiglu" (or 0 / 1); gate_mode: "switch" | "renorm" (or 0 / 1);
    capacity_factor <= 0: dropless; dtype: torch.float32 or torch.bfloat16;
    hidden (bf16 layers): "auto" (default) holds the hidden activation in fp16
    for batches of at least 1024 rows per expert and as a hi + lo pair of
    bf16 planes otherwise; "f16" and "bf16x2" force one of those; "bf16" is
    one bf16 plane (outside the parity bar; see include/moe.h).
    n_shared: shared experts every token visits; W1, W3, W2 then hold
    num_experts + n_shared experts, the shared ones last.
    """

    def __init__(self, num_experts: int, k: int, d: int, d_ff: int, act="swiglu", gate_mode="renorm",
                 capacity_factor: float = 0.0, dtype=torch.bfloat16, hidden="auto", n_shared: int = 0):
        self.E, self.k, self.d, self.d_ff = num_experts, k, d, d_ff
        self.act = ACT[act] if isinstance(act, str) else int(act)
        self.gate_mode = GATE[gate_mode] if isinstance(gate_mode, str) else int(gate_mode)
        self.capacity_factor = float(capacity_factor)
        self.dtype = dtype
        h = ctypes.c_void_p()
        check(lib().moe_create(num_experts, k, d, d_ff, self.act, self.gate_mode, self.capacity_factor,
                               DTYPE[dtype], ctypes.byref(h)))
        self._h = h
        self._ws = None
        self._bw = None  # backward scratch
        self.hidden = hidden
        check(lib().moe_set_hidden_precision(h, HIDDEN[hidden]))
        self.n_shared = int(n_shared)
        check(lib().moe_set_shared_experts(h, self.n_shared))

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and _lib._LIB is not None:
            _lib._LIB.moe_destroy(h)
            self._h = None

    def capacity(self, T: int) -> Optional[int]:
        c = lib().moe_capacity(self._h, T)
        return None if c < 0 else int(c)

    def workspace_bytes(self, T: int) -> int:
        return int(lib().moe_workspace_bytes(self._h, T))

    def workspace(self, T: int, device) -> torch.Tensor:
        n = self.workspace_bytes(T)
        if self._ws is None or self._ws.numel() < n or self._ws.device != torch.device(device):
            self._ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
        return self._ws

    def forward(self, x, W_r, b_r, W1, W3, W2, *, out=None, stats=None, workspace=None,
                debug: Optional[dict] = None, events=None, stream=None):
        """Run the layer.  Returns (y, expert_counts, dropped, aux_loss, z_loss) as device tensors.

        debug: optional dict of device tensors named like the fields of
        moe_debug (logits_in, logits_out, lse_out, topk_idx, topk_gate,
        dest_row, drop_mask, expert_offsets, y_f32).  events: optional list of
        2 * 6 torch.cuda.Event recorded around the kernel stages.
        """
        T = x.shape[0]
        dev = x.device
        y = out if out is not None else torch.empty((T, self.d), dtype=x.dtype, device=dev)
        if stats is None:
            stats = (torch.empty(self.E, dtype=torch.int32, device=dev),
                     torch.empty(1, dtype=torch.int32, device=dev),
                     torch.empty(1, dtype=torch.float32, device=dev),
                     torch.empty(1, dtype=torch.float32, device=dev))
        counts, dropped, aux, z = stats
        ws = workspace if workspace is not None else self.workspace(T, dev)
        dbg = _debug_struct(debug, events, stream)
        check(lib().moe_forward(
            self._h, T, _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(y),
            _ptr(counts), _ptr(dropped), _ptr(aux), _ptr(z), _ptr(ws), ws.numel(),
            None if dbg is None else ctypes.byref(dbg), _stream_handle(stream)))
        return y, counts, dropped, aux, z

    __call__ = forward

    def workspace_bytes_w4(self, T: int) -> int:
        return int(lib().moe_workspace_bytes_w4(self._h, T))

    def forward_w4(self, x, W_r, b_r, W1q, W3q, W2q, *, out=None, stats=None, workspace=None,
                   debug: Optional[dict] = None, events=None, stream=None):
        """The layer with 4-bit expert weights: W1q, W3q (None for ReLU), W2q are
        (codes, scales) pairs from quantize_int4.  Returns like forward()."""
        T = x.shape[0]
        dev = x.device
        y = out if out is not None else torch.empty((T, self.d), dtype=x.dtype, device=dev)
        if stats is None:
            stats = (torch.empty(self.E, dtype=torch.int32, device=dev),
                     torch.empty(1, dtype=torch.int32, device=dev),
                     torch.empty(1, dtype=torch.float32, device=dev),
                     torch.empty(1, dtype=torch.float32, device=dev))
        counts, dropped, aux, z = stats
        if workspace is None:
            n = self.workspace_bytes_w4(T)
            if self._ws is None or self._ws.numel() < n or self._ws.device != dev:
                self._ws = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
            workspace = self._ws
        dbg = _debug_struct(debug, events, stream)
        q3, s3 = (None, None) if W3q is None else W3q
        check(lib().moe_forward_w4(
            self._h, T, _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(W1q[0]), _ptr(W1q[1]), _ptr(q3), _ptr(s3),
            _ptr(W2q[0]), _ptr(W2q[1]), _ptr(y), _ptr(counts), _ptr(dropped), _ptr(aux), _ptr(z),
            _ptr(workspace), workspace.numel(), None if dbg is None else ctypes.byref(dbg), _stream_handle(stream)))
        return y, counts, dropped, aux, z

    def backward_workspace_bytes(self, T: int) -> int:
        return int(lib().moe_backward_workspace_bytes(self._h, T))

    def backward(self, x, W_r, b_r, W1, W3, W2, dy, *, aux_coef=0.0, z_coef=0.0, workspace=None,
                 bw_workspace=None, grads=None, stream=None) -> dict:
        """Gradients of <dy, y> + aux_coef * aux + z_coef * z for the last
        forward on ``workspace`` (default: this layer's own), routing held
        fixed.  Returns fp32 device tensors dx, dW_r, db_r (None without a
        bias), dW1, dW3 (None for ReLU), dW2; ``grads`` may supply them."""
        T, dev = x.shape[0], x.device
        ws = workspace if workspace is not None else self._ws
        if bw_workspace is None:
            n = self.backward_workspace_bytes(T)
            if self._bw is None or self._bw.numel() < n or self._bw.device != dev:
                self._bw = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
            bw_workspace = self._bw
        f32 = dict(dtype=torch.float32, device=dev)
        g = dict(grads or {})
        g.setdefault("dx", torch.empty((T, self.d), **f32))
        g.setdefault("dW_r", torch.empty(W_r.shape, **f32))
        g.setdefault("db_r", None if b_r is None else torch.empty(b_r.shape, **f32))
        g.setdefault("dW1", torch.empty(W1.shape, **f32))
        g.setdefault("dW3", None if W3 is None else torch.empty(W3.shape, **f32))
        g.setdefault("dW2", torch.empty(W2.shape, **f32))
        check(lib().moe_backward(
            self._h, T, _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(dy),
            float(aux_coef), float(z_coef), _ptr(g["dx"]), _ptr(g["dW_r"]), _ptr(g["db_r"]), _ptr(g["dW1"]),
            _ptr(g["dW3"]), _ptr(g["dW2"]), _ptr(ws), 0 if ws is None else ws.numel(), _ptr(bw_workspace),
            bw_workspace.numel(), _stream_handle(stream)))
        return g

    def balance_losses(self, T: int, workspace=None, out=None, stream=None) -> torch.Tensor:
        """The alternative balance statistics of the last forward on ``workspace``
        (default: this layer's own): a device tensor [aux over all k choices,
        CV of the assignment counts, cv^2 of the mean router probabilities]."""
        ws = workspace if workspace is not None else self._ws
        dev = ws.device if ws is not None else torch.device("cuda")
        out = out if out is not None else torch.empty(3, dtype=torch.float32, device=dev)
        check(lib().moe_balance_losses(self._h, T, _ptr(ws), _ptr(out), _stream_handle(stream)))
        return out

    def debug_buffers(self, T: int, device) -> dict:
        """Device tensors for every output field of moe_debug."""
        E, k = self.E, self.k
        return {
            "logits_out": torch.empty((T, E), dtype=torch.float32, device=device),
            "lse_out": torch.empty(T, dtype=torch.float32, device=device),
            "topk_idx": torch.empty((T, k), dtype=torch.int32, device=device),
            "topk_gate": torch.empty((T, k), dtype=torch.float32, device=device),
            "dest_row": torch.empty((T, k), dtype=torch.int32, device=device),
            "drop_mask": torch.empty((T, k), dtype=torch.uint8, device=device),
            "expert_offsets": torch.empty(E + 1, dtype=torch.int32, device=device),
            "y_f32": torch.empty((T, self.d), dtype=torch.float32, device=device),
        }


def quantize_int4(W: torch.Tensor, stream=None):
    """4-bit codes (int32 view of uint32 [rows][K / 8]) and bf16 scales
    [rows][K / 128] of a bf16 weight [..., K] (rows = every leading index),
    in the format of include/moe.h."""
    K = W.shape[-1]
    lead = W.shape[:-1]
    rows = W.numel() // K if K else 0
    codes = torch.empty(lead + (K // 8,), dtype=torch.int32, device=W.device)
    scales = torch.empty(lead + (K // 128,), dtype=torch.bfloat16, device=W.device)
    check(lib().moe_quantize_int4(_ptr(W.contiguous()), rows, K, _ptr(codes), _ptr(scales), _stream_handle(stream)))
    return codes, scales


def status(stream=None) -> None:
    """Synchronise the stream and raise MoEError if a kernel's bounded wait ran out."""
    check(lib().moe_status(_stream_handle(stream)))


def clear_status() -> None:
    check(lib().moe_clear_status())


def launch_count() -> int:
    return int(lib().moe_launch_count())


def selftest_timeout(limit_ns: int, stream=None) -> None:
    check(lib().moe_selftest_timeout(int(limit_ns), _stream_handle(stream)))
