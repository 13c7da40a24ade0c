"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Small seeded layers span several 128-row tiles, ragged tails in every
dimension, drops, ties, E in {1..256}, k in {1..8}; the router inputs are
dyadic so that fp32 logits are exact in any summation order and routing is
compared bit for bit through the whole path.  The full-size workloads are
checked on every token's routing and on sampled output rows.
"""
import zlib

import numpy as np
import pytest
import torch

from sparse_mixture_experts_gating_b200 import MoEError, MoELayer, clear_status, selftest_timeout, status
from sparse_mixture_experts_gating_b200.workloads import (ACT_RELU, ACT_SWIGLU, DTYPE_BF16, DTYPE_F32, GATE_RENORM,
                                                          GATE_SWITCH, WORKLOADS, Workload, make_inputs,
                                                          router_exactness_margin)
from tests._parity import (assert_gates_and_losses, assert_routing_equal, assert_y_close, host_inputs, layer_for,
                           run_gpu, run_oracle, sample_rows, y_errors)

pytestmark = pytest.mark.gpu

R, S = ACT_RELU, ACT_SWIGLU
SW, RN = GATE_SWITCH, GATE_RENORM
BF, F32 = DTYPE_BF16, DTYPE_F32

# name, T, d, E, k, d_ff, act, gate, cf, dtype, bias
SMALL = [
    ("tiny_fp32", 64, 32, 4, 2, 64, R, RN, 0.0, F32, None),
    ("swiglu_e8_k2", 1000, 256, 8, 2, 512, S, RN, 0.0, BF, None),
    ("switch_relu_drops", 999, 192, 16, 1, 384, R, SW, 1.0, BF, "normal"),
    ("k4_zipf_tails", 777, 136, 32, 4, 200, S, RN, 1.0, BF, "zipf"),
    ("single_expert", 300, 64, 1, 1, 128, R, RN, 0.0, BF, None),
    ("k_equals_E", 200, 64, 4, 4, 64, S, RN, 0.0, BF, None),
    ("e128_k8_cap", 500, 128, 128, 8, 64, S, RN, 2.0, BF, None),
    ("e256_switch", 300, 64, 256, 2, 64, R, SW, 0.0, BF, "normal"),
    ("capacity_one", 400, 64, 8, 2, 64, R, RN, 0.01, BF, None),
    ("one_token", 1, 64, 8, 2, 128, S, RN, 0.0, BF, None),
    ("fp32_swiglu_switch_cap", 301, 48, 6, 3, 40, S, SW, 1.5, F32, "normal"),
    ("fp32_relu_e1", 130, 24, 1, 1, 72, R, SW, 0.0, F32, None),
    ("long_k_ragged", 333, 1032, 4, 2, 1160, S, RN, 0.0, BF, None),
    ("decode_splitk", 3, 256, 8, 2, 1024, S, RN, 0.0, BF, None),          # K ranges of GEMM2 split
    ("decode_splitk_ragged", 5, 136, 4, 2, 1160, R, SW, 0.0, BF, "normal"),
    # grouped-GEMM wave tail: 1 < tiles / 148 < 2 ...
    ("wave_tail_relu", 600, 256, 8, 2, 4096, R, RN, 0.0, BF, None),
    # ... and few tiles over long K (K-range partials), k = 1 scatter epilogue, SwiGLU
    ("few_tiles_switch", 700, 512, 16, 1, 1024, R, SW, 1.25, BF, "normal"),
    ("few_tiles_long_k", 2, 2048, 4, 1, 256, R, RN, 0.0, BF, None),
    ("few_tiles_swiglu", 4, 1536, 8, 2, 384, S, RN, 0.0, BF, None),
    # shared experts (last field: n_shared): k = 2; k = 1 Switch with drops (the
    # combine path, dropped tokens keep the shared output); fp32; a small batch
    # whose second projection is split into K-range partials
    ("shared_k2_swiglu", 500, 128, 8, 2, 256, S, RN, 0.0, BF, None, 1),
    ("shared_switch_k1_drops", 400, 64, 16, 1, 128, R, SW, 0.5, BF, "normal", 2),
    ("shared_fp32", 120, 24, 4, 2, 40, S, RN, 1.0, F32, None, 1),
    ("shared_decode_splitk", 2, 256, 8, 2, 1024, S, RN, 0.0, BF, None, 1),
    # 33 <= T <= 64: pipeline stages hold 64 rows of A (T <= 32: 32 rows)
    ("ar64_swiglu", 48, 256, 8, 2, 512, S, RN, 0.0, BF, None),
    ("ar64_switch_shared", 61, 192, 4, 1, 384, R, SW, 1.0, BF, "normal", 1),
    # T <= 32 routes in two launches; here with fp32 rows (CUDA-core GEMMs), drops and a shared expert
    ("small_batch_fp32", 20, 40, 6, 2, 48, S, RN, 1.0, F32, "normal", 1),
    # 256 groups: 255 routed experts and one shared expert
    ("e255_shared", 300, 64, 255, 2, 64, R, RN, 0.0, BF, None, 1),
    # 66 router blocks x 256 experts: too many histogram entries for the fused
    # scan and dispatch, so the scan runs as its own launch (one block per
    # expert); the other cases above route in the fused launch
    ("e256_separate_scan", 2100, 64, 256, 1, 64, R, SW, 1.0, BF, "normal"),
    # 17..148 router tiles with d >= 4096: two K ranges per 128-token tile
    ("router_two_k_ranges", 2500, 4096, 64, 2, 256, S, RN, 2.0, BF, "zipf"),
]


def _small(case) -> Workload:
    name, T, d, E, k, d_ff, act, gate, cf, dt, bias = case[:11]
    n_shared = case[11] if len(case) > 11 else 0
    return Workload(name, T=T, d=d, E=E, k=k, d_ff=d_ff, act=act, gate=gate, capacity_factor=cf, dtype=dt,
                    bias=bias, dyadic=True, seed=4000 + zlib.crc32(name.encode()) % 1000, n_shared=n_shared)


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_layers_match_oracle(case):
    w = _small(case)
    inp = make_inputs(w, device="cuda")
    assert router_exactness_margin(inp["x"].float(), inp["W_r"], inp["b_r"]) < 2 ** 8
    g = run_gpu(w, inp)
    host = host_inputs(inp)
    o = run_oracle(w, host)
    np.testing.assert_array_equal(g["logits_out"], o["logits"])
    assert_routing_equal(g, o)
    assert_gates_and_losses(g, o)
    assert_y_close(w, g, o["y"])


SINGLE = [c for c in SMALL if c[9] == BF and c[0] in ("swiglu_e8_k2", "switch_relu_drops", "k4_zipf_tails",
                                                       "e128_k8_cap", "long_k_ragged", "wave_tail_relu",
                                                       "few_tiles_switch", "shared_switch_k1_drops",
                                                       "one_token", "ar64_swiglu")]


@pytest.mark.parametrize("case", SINGLE, ids=[c[0] for c in SINGLE])
def test_small_layers_single_bf16_hidden(case):
    """Hidden activation held in one bf16 plane: same routing, y within the
    mean bound against the plain oracle (this mode is outside the bar: see
    assert_y_close)."""
    w = _small(case)
    inp = make_inputs(w, device="cuda")
    g = run_gpu(w, inp, layer=layer_for(w, hidden="bf16"))
    host = host_inputs(inp)
    o = run_oracle(w, host)
    assert_routing_equal(g, o)
    assert_y_close(w, g, o["y"], single_plane_hidden=True)


F16 = [c for c in SMALL if c[9] == BF]


@pytest.mark.parametrize("case", F16, ids=[c[0] for c in F16])
def test_small_layers_f16_hidden(case):
    """Hidden activation in fp16 and the second projection on fp16 operands
    (an fp16 image of W2): routing bit-exact, y within the full bar."""
    w = _small(case)
    inp = make_inputs(w, device="cuda")
    g = run_gpu(w, inp, layer=layer_for(w, hidden="f16"))
    host = host_inputs(inp)
    o = run_oracle(w, host)
    assert_routing_equal(g, o)
    assert_gates_and_losses(g, o)
    assert_y_close(w, g, o["y"])


def test_f16_hidden_out_of_range_is_reported_and_context_survives():
    """A hidden value beyond the fp16 range (x scaled up 2^9) makes the fp16
    mode report MOE_ERR_RANGE; the status clears and the next call is fine."""
    w = _small(SMALL[1])
    inp = make_inputs(w, device="cuda")
    layer = layer_for(w, hidden="f16")
    clear_status()
    big = (inp["x"].float() * 512).to(torch.bfloat16)
    layer(big, inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"])
    with pytest.raises(MoEError) as ei:
        status()
    assert ei.value.code == 5
    clear_status()
    g = run_gpu(w, inp, layer=layer)
    o = run_oracle(w, host_inputs(inp))
    assert_routing_equal(g, o)
    assert_y_close(w, g, o["y"])


def test_ties_go_to_the_lower_expert_index():
    w = Workload("ties", T=257, d=64, E=8, k=3, d_ff=128, act=S, gate=RN, capacity_factor=0.0, dtype=BF,
                 dyadic=True, seed=77)
    inp = make_inputs(w, device="cuda")
    inp["W_r"][1] = inp["W_r"][0]   # experts 0 and 1 tie on every token
    inp["W_r"][5] = inp["W_r"][4]
    g = run_gpu(w, inp)
    host = host_inputs(inp)
    o = run_oracle(w, host)
    assert_routing_equal(g, o)
    both = (g["topk_idx"] == 0).any(1) & (g["topk_idx"] == 1).any(1)
    one = (g["topk_idx"] == 1).any(1) & ~(g["topk_idx"] == 0).any(1)
    assert both.any() and not one.any()  # expert 1 is never chosen without expert 0
    assert_y_close(w, g, o["y"])


def test_all_tokens_to_one_expert_with_capacity():
    w = Workload("collapsed", T=1500, d=128, E=8, k=1, d_ff=256, act=R, gate=SW, capacity_factor=1.0,
                 dtype=BF, dyadic=True, seed=91)
    inp = make_inputs(w, device="cuda")
    inp["b_r"] = torch.zeros(8, device="cuda")
    inp["b_r"][3] = 50.0
    g = run_gpu(w, inp)
    host = host_inputs(inp)
    o = run_oracle(w, host)
    assert (o["idx"][:, 0] == 3).all()
    assert_routing_equal(g, o)
    assert g["dropped"] == 1500 - 188  # capacity ceil(1500 / 8) = 188, first 188 tokens kept
    assert_y_close(w, g, o["y"])
    assert abs(g["aux"] - 8.0) < 1e-4


def test_zero_tokens():
    w = _small(SMALL[1])
    layer = layer_for(w)
    inp = make_inputs(w.with_(T=0), device="cuda")
    y, counts, dropped, aux, z = layer(inp["x"], inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"])
    status()
    assert y.shape == (0, w.d)
    assert counts.cpu().tolist() == [0] * w.E and dropped.item() == 0 and aux.item() == 0 and z.item() == 0


def test_deterministic_and_debug_hooks_do_not_change_results():
    w = _small(SMALL[3])
    inp = make_inputs(w, device="cuda")
    layer = layer_for(w)
    a = run_gpu(w, inp, debug=False, layer=layer)
    b = run_gpu(w, inp, debug=True, layer=layer)
    c = run_gpu(w, inp, debug=False, layer=layer)
    assert torch.equal(a["y_dev"].view(torch.int16), c["y_dev"].view(torch.int16))
    assert torch.equal(a["y_dev"].view(torch.int16), b["y_dev"].view(torch.int16))
    assert a["aux"] == b["aux"] == c["aux"] and a["z"] == c["z"]


def test_no_write_outside_outputs_and_workspace():
    w = _small(SMALL[2])
    inp = make_inputs(w, device="cuda")
    layer = layer_for(w)
    n = layer.workspace_bytes(w.T)
    ws = torch.full((n + 8192,), 0xA5, dtype=torch.uint8, device="cuda")
    ybuf = torch.full((w.T + 64, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    cbuf = torch.full((w.E + 16,), -7, dtype=torch.int32, device="cuda")
    stats = (cbuf[:w.E], torch.zeros(1, dtype=torch.int32, device="cuda"),
             torch.zeros(1, device="cuda"), torch.zeros(1, device="cuda"))
    layer(inp["x"], inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"], out=ybuf[:w.T], stats=stats,
          workspace=ws[:n])
    status()
    assert (ws[n:] == 0xA5).all()
    assert torch.isnan(ybuf[w.T:].float()).all()
    assert (cbuf[w.E:] == -7).all()
    assert not torch.isnan(ybuf[:w.T].float()).any()


def test_host_errors_leave_outputs_untouched():
    w = _small(SMALL[1])
    inp = make_inputs(w, device="cuda")
    layer = layer_for(w)
    y = torch.full((w.T, w.d), 3.0, dtype=torch.bfloat16, device="cuda")
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(MoEError) as ei:
        layer(inp["x"], inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"], out=y, workspace=small)
    assert ei.value.code == 1
    with pytest.raises(MoEError):
        layer(inp["x"], inp["W_r"], inp["b_r"], inp["W1"], None, inp["W2"], out=y)  # SwiGLU without W3
    torch.cuda.synchronize()
    assert (y.float() == 3.0).all()


def test_device_wait_timeout_is_reported_and_context_survives():
    clear_status()
    selftest_timeout(2_000_000)  # 2 ms on a flag nothing sets
    with pytest.raises(MoEError) as ei:
        status()
    assert ei.value.code == 4
    clear_status()
    status()
    w = _small(SMALL[1])  # the context is still usable
    inp = make_inputs(w, device="cuda")
    g = run_gpu(w, inp)
    o = run_oracle(w, host_inputs(inp))
    assert_routing_equal(g, o)


# ---------------------------------------------------------------- full-size workloads
FULL = ["switch_k1", "mixtral_prefill", "mixtral_decode_t1", "mixtral_decode_t16", "mixtral_decode_t64",
        "fine_grained", "fine_grained_shared"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_dyadic_routing_bit_exact(name):
    """Dyadic router inputs: every token's routing bit-exact through the whole path."""
    w = WORKLOADS[name].with_(dyadic=True)
    inp = make_inputs(w, device="cuda")
    assert router_exactness_margin(inp["x"].float(), inp["W_r"], inp["b_r"]) < 2 ** 8
    g = run_gpu(w, inp)
    host = host_inputs(inp)
    o_route = run_oracle(w, host, rows=[])
    np.testing.assert_array_equal(g["logits_out"], o_route["logits"])
    assert_routing_equal(g, o_route)
    assert_gates_and_losses(g, o_route)
    rows = sample_rows(w, o_route["kept"], n=24)
    o = run_oracle(w, host, rows=rows)
    assert_y_close(w, g, o["y"], rows=rows)


@pytest.mark.parametrize("name", FULL)
def test_full_size_identical_logits(name):
    """The workloads' own inputs; the oracle's fp32 logits are fed to both sides."""
    w = WORKLOADS[name]
    inp = make_inputs(w, device="cuda")
    host = host_inputs(inp)
    o_route = run_oracle(w, host, rows=[])
    g = run_gpu(w, inp, logits_in=torch.from_numpy(o_route["logits"]).cuda())
    assert_routing_equal(g, o_route)
    assert_gates_and_losses(g, o_route)
    rows = sample_rows(w, o_route["kept"], n=24, seed=1)
    o = run_oracle(w, host, rows=rows, logits=o_route["logits"])
    assert_y_close(w, g, o["y"], rows=rows)


@pytest.mark.parametrize("name", ["switch_k1", "mixtral_prefill", "fine_grained", "fine_grained_shared"])
def test_full_size_bench_configuration(name):
    """The launch the benchmark times (no debug hooks), on the workloads' own inputs.

    Router logits agree within the fp32 summation bound; every token whose
    choice is not within that bound of a tie routes identically; outputs of
    sampled rows routed identically match the oracle."""
    w = WORKLOADS[name]
    inp = make_inputs(w, device="cuda")
    layer = layer_for(w)
    plain = run_gpu(w, inp, debug=False, layer=layer)
    g = run_gpu(w, inp, debug=True, layer=layer)
    assert torch.equal(plain["y_dev"].view(torch.int16), g["y_dev"].view(torch.int16))
    host = host_inputs(inp)
    o_route = run_oracle(w, host, rows=[])
    # |fp32 sum - exact| <= d * 2^-24 * sum|w x| (+ bias rounding)
    bound = w.d * 2.0 ** -24 * (np.abs(host["x"]).astype(np.float64) @ np.abs(host["W_r"]).T.astype(np.float64))
    bound += 2.0 ** -23 * np.abs(o_route["logits"]).astype(np.float64) + 1e-30
    diff = np.abs(g["logits_out"].astype(np.float64) - o_route["logits"])
    assert (diff <= bound).all()
    srt = np.sort(o_route["logits"].astype(np.float64), axis=1)[:, ::-1]
    gaps = srt[:, :w.k] - srt[:, 1:w.k + 1]  # consecutive gaps among the top k+1
    clear = gaps.min(axis=1) > 2 * bound.max(axis=1)
    assert clear.mean() > 0.5
    assert (g["topk_idx"][clear] == o_route["idx"][clear]).all()
    assert g["counts"].sum() == w.T * w.k
    same = (g["topk_idx"] == o_route["idx"]).all(1) & (g["drop_mask"].astype(bool) == ~o_route["kept"]).all(1)
    rows = sample_rows(w, None, n=32, seed=2)
    rows = rows[same[rows]]
    assert len(rows) > 0
    o = run_oracle(w, host, rows=rows)
    assert_y_close(w, g, o["y"], rows=rows)


@pytest.mark.parametrize("name", ["switch_k1", "mixtral_prefill", "fine_grained", "mixtral_decode_t64"])
@pytest.mark.parametrize("hidden", ["f16", "bf16x2"])
def test_full_size_each_hidden_mode(name, hidden):
    """Both in-bar hidden modes forced at full size (identical logits): the
    automatic default picks one of them per batch, so each is checked on every
    shape class."""
    w = WORKLOADS[name]
    inp = make_inputs(w, device="cuda")
    host = host_inputs(inp)
    o_route = run_oracle(w, host, rows=[])
    g = run_gpu(w, inp, logits_in=torch.from_numpy(o_route["logits"]).cuda(), layer=layer_for(w, hidden=hidden))
    assert_routing_equal(g, o_route)
    rows = sample_rows(w, o_route["kept"], n=24, seed=4)
    o = run_oracle(w, host, rows=rows, logits=o_route["logits"])
    assert_y_close(w, g, o["y"], rows=rows)


@pytest.mark.parametrize("name", ["switch_k1", "mixtral_prefill", "fine_grained"])
def test_full_size_single_bf16_hidden(name):
    """Hidden activation in one bf16 plane at full size (identical logits):
    the mean bound against the plain oracle."""
    w = WORKLOADS[name]
    inp = make_inputs(w, device="cuda")
    host = host_inputs(inp)
    o_route = run_oracle(w, host, rows=[])
    g = run_gpu(w, inp, logits_in=torch.from_numpy(o_route["logits"]).cuda(), layer=layer_for(w, hidden="bf16"))
    assert_routing_equal(g, o_route)
    rows = sample_rows(w, o_route["kept"], n=24, seed=3)
    o = run_oracle(w, host, rows=rows, logits=o_route["logits"])
    assert_y_close(w, g, o["y"], rows=rows, single_plane_hidden=True)
