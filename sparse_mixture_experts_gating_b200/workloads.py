"""Seeded synthetic workloads for the MoE layer forward pass.

This module only draws random inputs of the right shapes and distributions.
It holds none of the layer's arithmetic: both the CUDA path and the CPU
oracle consume the tensors it returns.

Shapes follow the workloads the pages describe: a Switch-style k=1 layer
(Mixture of experts, rayaq.ca, section "Top-k gating", Switch bullet), a
Mixtral-shaped 8-expert top-2 SwiGLU layer (same page, "Total versus active
parameters" and "Implementation"), and a fine-grained many-expert layer
("2 out of 8 or 128", Mixture of Experts (MoE), inferensys.com
inference-optimization glossary, first paragraph), also with a shared expert
("Mixture of experts", rayaq.ca, "Total versus active parameters": shared
experts every token visits).

Distributions (no dataset exists for any of them):
  x ~ N(0, 1); router rows W_r ~ N(0, 1/d); expert weights ~ N(0, 1/fan_in)
  with fan_in = d for W1/W3 and d_ff for W2.  bf16 tensors are the
  round-to-nearest-even bf16 image of the fp32 draw.  W_r and the router bias
  stay fp32 (the router is computed in float32).
  Bias "normal": N(0, variance 0.5) per expert.
  Bias "zipf": a seeded permutation pi of the experts and
  bias[pi[r-1]] = -s * ln(r) for rank r = 1..E, s = 1.1, so that where the
  bias dominates, expert loads fall off like r^-s.

Dyadic variant (``dyadic=True``): x is rounded to multiples of 2^-6 and
clipped to [-4, 4]; W_r (and, for fp32 layers, every weight) is rounded to
multiples of 2^-10 and clipped to |w| <= 1 - 2^-10; the bias is rounded to
multiples of 2^-10.  Then every product w*x is a multiple of 2^-16, and as
long as sum_c |w_c x_c| + |b| < 2^8 every partial sum of a router logit is
exactly representable in fp32, whatever the summation order.
``router_exactness_margin`` reports that bound so tests can assert it.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional

import torch

ACT_RELU, ACT_SWIGLU = 0, 1
GATE_SWITCH, GATE_RENORM = 0, 1
DTYPE_F32, DTYPE_BF16 = 0, 1


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    d_ff: int
    act: int
    gate: int
    capacity_factor: float  # <= 0 means dropless
    dtype: int
    bias: Optional[str] = None  # None | "normal" | "zipf"
    dyadic: bool = False
    x_rows_of: Optional[str] = None  # take x as the first T rows of this workload's x
    seed: int = 1234
    n_shared: int = 0  # shared experts every token visits (weights follow the routed experts')

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_fp32", T=64, d=32, E=4, k=2, d_ff=64, act=ACT_RELU,
                 gate=GATE_RENORM, capacity_factor=0.0, dtype=DTYPE_F32,
                 dyadic=True, seed=1234),
        Workload("switch_k1", T=8192, d=768, E=64, k=1, d_ff=3072, act=ACT_RELU,
                 gate=GATE_SWITCH, capacity_factor=1.25, dtype=DTYPE_BF16,
                 bias="normal", seed=1235),
        Workload("mixtral_prefill", T=8192, d=4096, E=8, k=2, d_ff=14336,
                 act=ACT_SWIGLU, gate=GATE_RENORM, capacity_factor=0.0,
                 dtype=DTYPE_BF16, seed=1236),
        Workload("mixtral_decode_t1", T=1, d=4096, E=8, k=2, d_ff=14336,
                 act=ACT_SWIGLU, gate=GATE_RENORM, capacity_factor=0.0,
                 dtype=DTYPE_BF16, x_rows_of="mixtral_prefill", seed=1236),
        Workload("mixtral_decode_t16", T=16, d=4096, E=8, k=2, d_ff=14336,
                 act=ACT_SWIGLU, gate=GATE_RENORM, capacity_factor=0.0,
                 dtype=DTYPE_BF16, x_rows_of="mixtral_prefill", seed=1236),
        Workload("mixtral_decode_t64", T=64, d=4096, E=8, k=2, d_ff=14336,
                 act=ACT_SWIGLU, gate=GATE_RENORM, capacity_factor=0.0,
                 dtype=DTYPE_BF16, x_rows_of="mixtral_prefill", seed=1236),
        Workload("fine_grained", T=16384, d=2048, E=128, k=4, d_ff=768,
                 act=ACT_SWIGLU, gate=GATE_RENORM, capacity_factor=2.0,
                 dtype=DTYPE_BF16, bias="zipf", seed=1238),
        # the fine-grained layer plus one shared expert of the same shape
        # ("many small experts plus shared experts every token visits")
        Workload("fine_grained_shared", T=16384, d=2048, E=128, k=4, d_ff=768,
                 act=ACT_SWIGLU, gate=GATE_RENORM, capacity_factor=2.0,
                 dtype=DTYPE_BF16, bias="zipf", seed=1238, n_shared=1),
    ]
}

# stream ids: one independent generator per tensor
_SID = {"x": 1, "W_r": 2, "b_r": 3, "W1": 4, "W3": 5, "W2": 6, "perm": 7}


def _gen(device, seed: int, stream: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 64 + _SID[stream])
    return g


def _normal(shape, std, device, seed, stream):
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(0.0, std, generator=_gen(device, seed, stream))
    return t


def _round_to_grid(t: torch.Tensor, log2_step: int, bound: float) -> torch.Tensor:
    step = 2.0 ** log2_step
    return torch.clamp(torch.round(t / step) * step, -bound, bound)


def torch_dtype(code: int):
    return torch.float32 if code == DTYPE_F32 else torch.bfloat16


def make_inputs(w: Workload, device="cpu", weights=True, x_rows: Optional[int] = None):
    """Draw the layer inputs of workload ``w`` on ``device``.

    Returns a dict with x [T][d], W_r [E][d] (fp32), b_r [E] (fp32) or None,
    W1 [E + n_shared][d_ff][d], W3 [E + n_shared][d_ff][d] (SwiGLU only, else
    None), W2 [E + n_shared][d][d_ff] (the shared experts last).  x and the
    expert weights have the workload's dtype.
    """
    dev = torch.device(device)
    dt = torch_dtype(w.dtype)
    src_T = WORKLOADS[w.x_rows_of].T if w.x_rows_of else w.T
    rows = w.T if x_rows is None else x_rows
    x = _normal((max(src_T, w.T), w.d), 1.0, dev, w.seed, "x")[:rows]
    W_r = _normal((w.E, w.d), 1.0 / math.sqrt(w.d), dev, w.seed, "W_r")
    b_r = None
    if w.bias == "normal":
        b_r = _normal((w.E,), math.sqrt(0.5), dev, w.seed, "b_r")
    elif w.bias == "zipf":
        perm = torch.randperm(w.E, generator=_gen("cpu", w.seed, "perm"))
        ranks = torch.arange(1, w.E + 1, dtype=torch.float64)
        b = torch.empty(w.E, dtype=torch.float64)
        b[perm] = -1.1 * torch.log(ranks)
        b_r = b.to(torch.float32).to(dev)
    if w.dyadic:
        x = _round_to_grid(x, -6, 4.0)
        W_r = _round_to_grid(W_r, -10, 1.0 - 2.0 ** -10)
        if b_r is not None:
            b_r = _round_to_grid(b_r, -10, 64.0)
    out = {"x": x.to(dt).contiguous(), "W_r": W_r.contiguous(), "b_r": b_r,
           "W1": None, "W3": None, "W2": None}
    if weights:
        ne = w.E + w.n_shared
        W1 = _normal((ne, w.d_ff, w.d), 1.0 / math.sqrt(w.d), dev, w.seed, "W1")
        W2 = _normal((ne, w.d, w.d_ff), 1.0 / math.sqrt(w.d_ff), dev, w.seed, "W2")
        W3 = None
        if w.act == ACT_SWIGLU:
            W3 = _normal((ne, w.d_ff, w.d), 1.0 / math.sqrt(w.d), dev, w.seed, "W3")
        if w.dyadic and w.dtype == DTYPE_F32:
            W1 = _round_to_grid(W1, -10, 1.0 - 2.0 ** -10)
            W2 = _round_to_grid(W2, -10, 1.0 - 2.0 ** -10)
            if W3 is not None:
                W3 = _round_to_grid(W3, -10, 1.0 - 2.0 ** -10)
        out["W1"] = W1.to(dt).contiguous()
        out["W2"] = W2.to(dt).contiguous()
        out["W3"] = None if W3 is None else W3.to(dt).contiguous()
    return out


def router_exactness_margin(x: torch.Tensor, W_r: torch.Tensor, b_r=None) -> float:
    """max over (token, expert) of sum_c |W_r[e,c] x[t,c]| + |b[e]|.

    Below 2^8 (with the dyadic grids above) every partial sum of every router
    logit is exact in fp32, so logits do not depend on summation order.
    """
    s = x.double().abs() @ W_r.double().abs().t()
    if b_r is not None:
        s = s + b_r.double().abs()
    return float(s.max()) if s.numel() else 0.0
