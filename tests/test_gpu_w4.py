"""4-bit expert weights (moe_quantize_int4, moe_forward_w4) against the oracle.

The quantizer's codes and scales are integer / exactly representable results
of float32 decisions, so they must equal the oracle's (oracle.moe_oracle
quantize_int4 and pack_int4, the same rule in float32) bit for bit.  The
4-bit forward must equal the layer computed by the oracle with the
dequantized weights (exact in bf16): routing bit-exact on dyadic router
inputs, y within the bf16 bar (max|dy| <= 1e-2 RMS, mean relative 2e-3).
Batches of at most 64 tokens run the few-row products (warp MMAs fed from
registers; groups above 32 / 16 rows in several chunks), larger ones the
tcgen05 grouped GEMM; the cases cover both.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle.moe_oracle as M
from sparse_mixture_experts_gating_b200 import MoEError, quantize_int4, status
from sparse_mixture_experts_gating_b200.workloads import (ACT_RELU, ACT_SWIGLU, DTYPE_BF16, GATE_RENORM,
                                                          GATE_SWITCH, WORKLOADS, Workload, make_inputs)
from tests._parity import assert_gates_and_losses, assert_routing_equal, assert_y_close, layer_for, np32, sample_rows

pytestmark = pytest.mark.gpu

R, S = ACT_RELU, ACT_SWIGLU
SW, RN = GATE_SWITCH, GATE_RENORM


def _words(codes: torch.Tensor) -> np.ndarray:
    return codes.cpu().numpy().view(np.uint32)


def test_quantizer_matches_the_oracle_bit_for_bit():
    gen = torch.Generator(device="cuda").manual_seed(17)
    W = (torch.randn(384, 1024, device="cuda", generator=gen) * 0.02)
    W[5, 128:256] = 0.0                        # an all-zero group: scale 0, codes 8
    W[7, :128] = torch.arange(128, device="cuda") - 64.0  # integer values: many exact halves after division
    W[9, :128] *= 1e-30                        # tiny values (subnormal scale region)
    W = W.to(torch.bfloat16)
    codes, scales = quantize_int4(W)
    status()
    q, s = M.quantize_int4(W.float().cpu().numpy())
    np.testing.assert_array_equal(_words(codes).reshape(-1), M.pack_int4(q))
    np.testing.assert_array_equal(scales.float().cpu().numpy().reshape(-1), M.tile_scales(s))
    assert (s.view(np.uint32) & 0x7FFFF == 0).all()  # at most 5 significant bits


def test_quantizer_round_trip_error_is_at_most_half_a_step():
    W = (torch.randn(128, 512, device="cuda", generator=torch.Generator(device="cuda").manual_seed(3)) * 0.05)
    W = W.to(torch.bfloat16)
    codes, scales = quantize_int4(W)
    status()
    Wd = M.dequantize_int4(_words(codes), scales.float().cpu().numpy(), 128, 512)
    s_rows = scales.float().cpu().numpy().reshape(1, 4, 128).transpose(0, 2, 1).reshape(128, 4)
    step = np.repeat(s_rows.astype(np.float64), 128, axis=1)
    assert (np.abs(Wd - W.float().cpu().numpy()) <= 0.5 * step + 1e-30).all()


class Dequant:
    """Per-expert dequantized host copies of 4-bit device weights [G][rows][K] (lazy)."""

    def __init__(self, pair):
        self.codes, self.scales = pair
        self.cache = {}

    def __getitem__(self, e):
        if e not in self.cache:
            rows, K = self.codes.shape[1], self.codes.shape[2] * 8
            self.cache[e] = M.dequantize_int4(_words(self.codes[e]), self.scales[e].float().cpu().numpy(), rows, K)
        return self.cache[e]

    def __len__(self):
        return self.codes.shape[0]


class _Shift:
    def __init__(self, d, E, n):
        self.d, self.E, self.n = d, E, n

    def __len__(self):
        return self.n

    def __getitem__(self, s):
        return self.d[self.E + s]


def _quantized(inp):
    return {k: (None if inp[k] is None else quantize_int4(inp[k])) for k in ("W1", "W3", "W2")}


def _run_w4(w, inp, qw, debug=True, logits_in=None):
    layer = layer_for(w)
    dbg = layer.debug_buffers(w.T, inp["x"].device) if debug else None
    if logits_in is not None:
        dbg = dbg or {}
        dbg["logits_in"] = logits_in
    y, counts, dropped, aux, z = layer.forward_w4(inp["x"], inp["W_r"], inp["b_r"], qw["W1"], qw["W3"], qw["W2"],
                                                  debug=dbg)
    status()
    g = {"y_dev": y, "y": np32(y), "counts": counts.cpu().numpy(), "dropped": int(dropped.item()),
         "aux": float(aux.item()), "z": float(z.item())}
    for key, t in (dbg or {}).items():
        if key != "logits_in":
            g[key] = t.cpu().numpy() if t.dtype != torch.float32 else np32(t)
    return g


def _oracle_w4(w, inp, qw, rows=None, logits=None):
    D1, D2 = Dequant(qw["W1"]), Dequant(qw["W2"])
    D3 = None if qw["W3"] is None else Dequant(qw["W3"])
    shared = None
    if w.n_shared:
        shared = (_Shift(D1, w.E, w.n_shared), None if D3 is None else _Shift(D3, w.E, w.n_shared),
                  _Shift(D2, w.E, w.n_shared))
    return M.moe_forward(np32(inp["x"]), np32(inp["W_r"]), np32(inp["b_r"]), D1, D3, D2, k=w.k, gate_mode=w.gate,
                         act=w.act, capacity_factor=w.capacity_factor, rows=rows, logits=logits, shared=shared)


# name, T, d, E, k, d_ff, act, gate, cf, bias, n_shared
CASES = [
    ("w4_one_token", 1, 256, 8, 2, 384, S, RN, 0.0, None, 0),
    ("w4_t16", 16, 512, 8, 2, 1024, S, RN, 0.0, None, 0),
    ("w4_t33_relu_switch", 33, 256, 16, 1, 640, R, SW, 1.0, "normal", 0),
    ("w4_t64", 64, 384, 8, 2, 768, S, RN, 0.0, None, 0),
    ("w4_shared", 40, 256, 4, 2, 256, S, RN, 1.0, None, 1),
    # groups of more than 64 rows: several n-tiles per expert
    ("w4_large_groups", 300, 256, 4, 2, 384, S, RN, 0.0, "normal", 0),
    # few-row products: 12 rows per group (two n-tiles of the first projection,
    # three of the second), odd m-tile counts (a unit with one slot), ReLU
    ("w4_small_relu_odd_tiles", 12, 384, 2, 2, 640, R, RN, 0.0, "normal", 0),
    # few-row products with a shared expert (a group of every token)
    ("w4_small_shared", 5, 256, 8, 2, 384, S, RN, 0.0, None, 1),
    # few-row products with capacity drops (at most 8 rows per expert)
    ("w4_small_capacity", 16, 512, 4, 2, 256, S, RN, 1.0, None, 0),
    # few-row products over a long K range (d_ff 2048: 16 scale groups)
    ("w4_small_long_k", 3, 1024, 16, 4, 2048, S, RN, 0.0, "normal", 0),
    # few-row products with groups of 64 rows (two chunks of the first
    # projection, four of the second) and a shared expert of 64 rows
    ("w4_small_chunks", 64, 256, 2, 2, 384, S, RN, 0.0, None, 1),
    # the tcgen05 grouped GEMM just above the few-row range, ReLU, shared expert
    ("w4_tc_t65_relu_shared", 65, 256, 4, 2, 256, R, RN, 0.0, "normal", 1),
    ("w4_tc_t128", 128, 384, 8, 2, 640, S, RN, 1.0, None, 0),
    # few-row products over many groups (64 experts, top-4: up to 64 groups with rows)
    ("w4_small_many_experts", 32, 256, 64, 4, 256, S, RN, 0.0, "zipf", 0),
    # few-row products with capacity drops and a shared expert, Switch gate
    ("w4_small_drops_shared", 48, 384, 8, 1, 384, R, SW, 0.5, "normal", 1),
]


def _w(case) -> Workload:
    name, T, d, E, k, d_ff, act, gate, cf, bias, ns = case
    return Workload(name, T=T, d=d, E=E, k=k, d_ff=d_ff, act=act, gate=gate, capacity_factor=cf, dtype=DTYPE_BF16,
                    bias=bias, dyadic=True, seed=7000 + zlib.crc32(name.encode()) % 1000, n_shared=ns)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_w4_layers_match_oracle_with_dequantized_weights(case):
    w = _w(case)
    inp = make_inputs(w, device="cuda")
    qw = _quantized(inp)
    g = _run_w4(w, inp, qw)
    o = _oracle_w4(w, inp, qw)
    np.testing.assert_array_equal(g["logits_out"], o["logits"])
    assert_routing_equal(g, o)
    assert_gates_and_losses(g, o)
    assert_y_close(w, g, o["y"])


@pytest.mark.parametrize("name", ["mixtral_decode_t1", "mixtral_decode_t16", "mixtral_decode_t64"])
def test_w4_full_size_decode(name):
    """The Mixtral-shaped decode layers with their weights quantized: every
    token's routing and every output row against the oracle (dequantized
    weights; identical logits)."""
    w = WORKLOADS[name]
    inp = make_inputs(w, device="cuda")
    qw = _quantized(inp)
    del inp["W1"], inp["W3"], inp["W2"]
    inp.update(W1=None, W3=None, W2=None)
    o_route = M.moe_forward(np32(inp["x"]), np32(inp["W_r"]), None, [np.zeros((1, w.d))] * w.E, None,
                            [np.zeros((w.d, 1))] * w.E, k=w.k, gate_mode=w.gate, act=w.act,
                            capacity_factor=w.capacity_factor, rows=[])
    g = _run_w4(w, inp, qw, logits_in=torch.from_numpy(o_route["logits"]).cuda())
    assert_routing_equal(g, o_route)
    rows = sample_rows(w, None, n=16)
    o = _oracle_w4(w, inp, qw, rows=rows, logits=o_route["logits"])
    assert_y_close(w, g, o["y"], rows=rows)


def test_w4_empty_batch():
    """T = 0: no launch of the expert products; zeroed counts and losses."""
    w = _w(("w4_empty", 0, 256, 8, 2, 256, S, RN, 0.0, None, 0))
    inp = make_inputs(Workload("w4_empty_src", T=1, d=256, E=8, k=2, d_ff=256, act=S, gate=RN, capacity_factor=0.0,
                               dtype=DTYPE_BF16, dyadic=True, seed=3), device="cuda")
    qw = _quantized(inp)
    layer = layer_for(w)
    x = inp["x"][:0]
    y, counts, dropped, aux, z = layer.forward_w4(x, inp["W_r"], inp["b_r"], qw["W1"], qw["W3"], qw["W2"])
    status()
    assert y.shape == (0, 256)
    assert int(counts.sum().item()) == 0 and int(dropped.item()) == 0
    assert float(aux.item()) == 0.0 and float(z.item()) == 0.0


def test_w4_rejects_dimensions_off_the_group_size():
    w = Workload("w4_bad", T=8, d=136, E=4, k=2, d_ff=256, act=S, gate=RN, capacity_factor=0.0, dtype=DTYPE_BF16,
                 dyadic=True, seed=5)
    inp = make_inputs(w, device="cuda")
    layer = layer_for(w)
    fake = (torch.zeros(8, dtype=torch.int32, device="cuda"), torch.zeros(8, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(MoEError) as ei:
        layer.forward_w4(inp["x"], inp["W_r"], inp["b_r"], fake, fake, fake)
    assert ei.value.code == 2
    with pytest.raises(MoEError):
        quantize_int4(inp["W1"])  # K = 136
