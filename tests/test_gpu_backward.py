"""Parity of the backward pass (moe_backward through the C ABI) with the
backward oracle (oracle/moe_backward.py, pinned by finite differences).

Small seeded layers with dyadic router inputs, so that the routing of the
forward pass is the oracle's (checked), then every gradient tensor is
compared element by element.  Tolerance, per tensor: max|got - ref| <=
2e-4 * max|ref|.  The kernels accumulate in fp32 sums of at most a few
thousand products (relative error about sqrt(K) * 2^-24, below 1e-5 of the
operands' scale); the router's gradient subtracts <dp, p> from dp, which
loses a few more bits where the two are close.  A wrong term or sign moves a
tensor by O(1) of its scale.
"""
import zlib

import numpy as np
import pytest
import torch

from oracle import moe_backward as OB
from sparse_mixture_experts_gating_b200 import status
from sparse_mixture_experts_gating_b200.workloads import (ACT_RELU, ACT_SWIGLU, DTYPE_BF16, DTYPE_F32, GATE_RENORM,
                                                          GATE_SWITCH, Workload, make_inputs)
from tests._parity import layer_for, np32

pytestmark = pytest.mark.gpu

R, S = ACT_RELU, ACT_SWIGLU
SW, RN = GATE_SWITCH, GATE_RENORM
BF, F32 = DTYPE_BF16, DTYPE_F32
AUX, ZC = 0.37, 0.21
TOL = 2e-4

# name, T, d, E, k, d_ff, act, gate, cf, dtype, bias, n_shared
CASES = [
    ("switch_relu_drops_bf16", 300, 64, 8, 1, 96, R, SW, 1.0, BF, "normal", 0),
    ("renorm_swiglu_bf16", 257, 48, 6, 2, 80, S, RN, 0.0, BF, None, 0),
    ("switch_k2_swiglu_fp32", 130, 40, 5, 2, 56, S, SW, 1.25, F32, "normal", 0),
    ("shared_swiglu_drops_bf16", 150, 64, 4, 2, 64, S, RN, 1.0, BF, None, 1),
    ("small_batch_bf16", 20, 64, 8, 2, 64, S, RN, 0.0, BF, "normal", 0),  # one launch routes T <= 32
    ("e32_k4_zipf_relu", 200, 32, 32, 4, 40, R, RN, 1.0, BF, "zipf", 0),
    # at size: T >= 1024 sums dW_r over four or more token chunks; d >= 256 and
    # d_ff >= 512 give several n-tiles and k-blocks in every product
    ("chunks_relu_drops", 1100, 256, 8, 1, 512, R, SW, 1.25, BF, "normal", 0),
    ("chunks_swiglu_k2", 1536, 384, 8, 2, 640, S, RN, 0.0, BF, None, 0),
    # skewed loads: the largest expert group (and so the padded K of the
    # weight-gradient products) is well above 512 rows
    ("skewed_kpad_swiglu", 2048, 256, 4, 1, 512, S, SW, 0.0, BF, "zipf", 0),
    ("chunks_shared_fp32", 1030, 64, 4, 2, 96, S, RN, 1.0, F32, "normal", 1),
]


def _w(case) -> Workload:
    name, T, d, E, k, d_ff, act, gate, cf, dt, bias, ns = case
    return Workload(name, T=T, d=d, E=E, k=k, d_ff=d_ff, act=act, gate=gate, capacity_factor=cf, dtype=dt,
                    bias=bias, dyadic=True, seed=6000 + zlib.crc32(name.encode()) % 1000, n_shared=ns)


def _run(w: Workload):
    inp = make_inputs(w, device="cuda")
    layer = layer_for(w)
    dbg = layer.debug_buffers(w.T, inp["x"].device)
    layer(inp["x"], inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"], debug=dbg)
    gen = torch.Generator().manual_seed(99)
    dy = torch.randn(w.T, w.d, generator=gen).to(inp["x"].dtype).to(inp["x"].device)
    g = layer.backward(inp["x"], inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"], dy,
                       aux_coef=AUX, z_coef=ZC)
    status()
    return inp, layer, dbg, dy, g


def _oracle(w: Workload, inp: dict, dy):
    E = w.E
    W1, W2 = np32(inp["W1"]), np32(inp["W2"])
    W3 = None if inp["W3"] is None else np32(inp["W3"])
    shared = None
    if w.n_shared:
        shared = (W1[E:], None if W3 is None else W3[E:], W2[E:])
    return OB.moe_backward(np32(inp["x"]), np32(inp["W_r"]), np32(inp["b_r"]), W1[:E],
                           None if W3 is None else W3[:E], W2[:E], np32(dy), k=w.k, gate_mode=w.gate, act=w.act,
                           capacity_factor=w.capacity_factor, aux_coef=AUX, z_coef=ZC, shared=shared)


def _close(name, got, ref):
    got = np.asarray(got, np.float64)
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    err = float(np.abs(got - ref).max()) if ref.size else 0.0
    assert err <= TOL * scale + 1e-30, f"{name}: max|d| {err:.3e} vs scale {scale:.3e}"


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(case):
    w = _w(case)
    inp, _, dbg, dy, g = _run(w)
    o = _oracle(w, inp, dy)
    np.testing.assert_array_equal(dbg["topk_idx"].cpu().numpy(), o["idx"])
    np.testing.assert_array_equal(dbg["drop_mask"].cpu().numpy().astype(bool), ~o["kept"])
    if w.capacity_factor > 0 and case[0] != "small_batch_bf16":
        assert not o["kept"].all()
    E = w.E
    _close("dx", np32(g["dx"]), o["dx"])
    _close("dW_r", np32(g["dW_r"]), o["dW_r"])
    if inp["b_r"] is not None:
        _close("db_r", np32(g["db_r"]), o["db_r"])
    _close("dW1", np32(g["dW1"])[:E], o["dW1"])
    _close("dW2", np32(g["dW2"])[:E], o["dW2"])
    if w.act == S:
        _close("dW3", np32(g["dW3"])[:E], o["dW3"])
    if w.n_shared:
        _close("dW1s", np32(g["dW1"])[E:], o["dW1s"])
        _close("dW2s", np32(g["dW2"])[E:], o["dW2s"])
        if w.act == S:
            _close("dW3s", np32(g["dW3"])[E:], o["dW3s"])


def test_skewed_case_pads_k_beyond_512():
    w = _w([c for c in CASES if c[0] == "skewed_kpad_swiglu"][0])
    inp, _, dbg, dy, g = _run(w)
    counts = np.bincount(dbg["topk_idx"].cpu().numpy().ravel(), minlength=w.E)
    assert counts.max() > 512


def test_full_size_switch_backward_matches_oracle():
    """The Switch workload at full size (T 8192, d 768, 64 experts, ReLU 3072,
    capacity 1.25) with dyadic router inputs, every element of every gradient
    tensor against the backward oracle.

    The ReLU derivative is a floating-point decision: relu'(a) jumps from 0 to 1
    at a = 0, and the kernel takes it on its fp32 tensor-core sum of w1 x while
    the oracle takes it on the exact value.  Where |a| lies within the fp32
    summation bound of 0 ((d / 16 + 16) 2^-23 sum_c |w1_c x_c|: fp32 partial
    sums of 16 exact products, one rounding each, counted at double the unit
    roundoff) either decision is correct, and the gradients that see it (dx of
    that token, row f of that expert's dW1) may differ from the oracle's by
    the whole term |U_tf| |W1[f]| (resp. |U_tf| |x_t|), U_tf = g_t (W2^T dy_t)_f;
    they are checked to within that allowance, everything else to the usual
    bound.  dW2, dW_r and db_r see relu(a) itself, continuous there."""
    from sparse_mixture_experts_gating_b200.workloads import WORKLOADS
    w = WORKLOADS["switch_k1"].with_(dyadic=True)
    inp, _, dbg, dy, g = _run(w)
    o = _oracle(w, inp, dy)
    np.testing.assert_array_equal(dbg["topk_idx"].cpu().numpy(), o["idx"])
    np.testing.assert_array_equal(dbg["drop_mask"].cpu().numpy().astype(bool), ~o["kept"])
    assert not o["kept"].all()
    x = np32(inp["x"]).astype(np.float64)
    dyh = np32(dy).astype(np.float64)
    gate = dbg["topk_gate"].cpu().numpy().astype(np.float64)[:, 0]
    allow_dx = np.zeros((w.T, w.d))
    allow_dw1 = np.zeros((w.E, w.d_ff, w.d))
    n_near_tokens = 0
    for e in range(w.E):
        ts = np.nonzero((o["idx"][:, 0] == e) & o["kept"][:, 0])[0]
        if ts.size == 0:
            continue
        W1e = inp["W1"][e].float().cpu().numpy().astype(np.float64)
        W2e = inp["W2"][e].float().cpu().numpy().astype(np.float64)
        a = x[ts] @ W1e.T
        bound = (w.d / 16 + 16) * 2.0 ** -23 * (np.abs(x[ts]) @ np.abs(W1e).T)
        near = np.abs(a) <= bound
        rows = np.nonzero(near.any(axis=1))[0]
        n_near_tokens += rows.size
        if rows.size == 0:
            continue
        U = np.abs(gate[ts[rows], None] * (dyh[ts[rows]] @ W2e)) * near[rows]  # [n][d_ff], 0 where sure
        allow_dx[ts[rows]] = U @ np.abs(W1e)
        allow_dw1[e] = U.T @ np.abs(x[ts[rows]])
    assert n_near_tokens < 0.5 * w.T

    def close_with(name, got, ref, allow):
        scale = float(np.abs(ref).max())
        err = np.abs(np.asarray(got, np.float64) - ref)
        assert (err <= TOL * scale + allow).all(), f"{name}: max excess {(err - TOL * scale - allow).max():.3e}"

    close_with("dx", np32(g["dx"]), o["dx"], allow_dx)
    close_with("dW1", np32(g["dW1"])[:w.E], o["dW1"], allow_dw1)
    sure = allow_dx.max(axis=1) == 0
    _close("dx (tokens whose ReLU decisions are unique)", np32(g["dx"])[sure], o["dx"][sure])
    for key in ("dW_r", "db_r", "dW2"):
        _close(key, np32(g[key]), o[key])


def test_backward_is_deterministic():
    w = _w(CASES[1])
    inp, layer, _, dy, g1 = _run(w)
    g2 = layer.backward(inp["x"], inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"], dy,
                        aux_coef=AUX, z_coef=ZC)
    status()
    for key in ("dx", "dW_r", "dW1", "dW3", "dW2"):
        assert torch.equal(g1[key], g2[key]), key


def test_backward_zero_tokens():
    w = _w(CASES[0])
    inp = make_inputs(w, device="cuda")
    layer = layer_for(w)
    x0 = inp["x"][:0]
    layer(x0, inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"])
    grads = {"dW1": torch.full(inp["W1"].shape, 7.0, device="cuda"),
             "dW2": torch.full(inp["W2"].shape, 7.0, device="cuda")}
    g = layer.backward(x0, inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"], x0, grads=grads)
    status()
    for key in ("dW_r", "db_r", "dW1", "dW2"):
        assert not torch.any(g[key]), key


def test_expert_no_token_chooses_gets_zero_weight_gradients():
    """An expert that no token routes to has an empty group: the weight
    gradients' products run none of its k-blocks, and its dW1 / dW2 rows must
    come out exactly zero (the oracle's sum over no rows), the rest as usual.
    A router bias of -64 on expert 3 (dyadic, so the logits stay exact) keeps
    every token away from it."""
    w = _w(CASES[0])
    inp = make_inputs(w, device="cuda")
    inp["b_r"][3] = -64.0
    layer = layer_for(w)
    dbg = layer.debug_buffers(w.T, inp["x"].device)
    layer(inp["x"], inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"], debug=dbg)
    gen = torch.Generator().manual_seed(99)
    dy = torch.randn(w.T, w.d, generator=gen).to(inp["x"].dtype).to(inp["x"].device)
    g = layer.backward(inp["x"], inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"], dy,
                       aux_coef=AUX, z_coef=ZC)
    status()
    idx = dbg["topk_idx"].cpu().numpy()
    assert not (idx == 3).any()
    o = _oracle(w, inp, dy)
    np.testing.assert_array_equal(idx, o["idx"])
    assert not np.any(np32(g["dW1"])[3]) and not np.any(np32(g["dW2"])[3])
    E = w.E
    _close("dx", np32(g["dx"]), o["dx"])
    _close("dW_r", np32(g["dW_r"]), o["dW_r"])
    _close("dW1", np32(g["dW1"])[:E], o["dW1"])
    _close("dW2", np32(g["dW2"])[:E], o["dW2"])
