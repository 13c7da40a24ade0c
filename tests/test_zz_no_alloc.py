"""moe_forward_static: the entry point for callers that cannot allocate
device memory (for instance a plug-in whose host framework owns every device
allocation), which takes its scratch from a fixed array inside the library.

Called through the C ABI and checked against moe_forward (caller workspace)
on two calls in a row with different inputs.  Both entry points run the same
deterministic kernels on the same inputs, so the results must agree bit for
bit: a stale value read from the shared scratch would show up as a
difference.  This file is collected last, so a run that stops at the first
failure has run every other test already.
"""
import ctypes

import pytest
import torch

from sparse_mixture_experts_gating_b200 import MoELayer, status
from sparse_mixture_experts_gating_b200._lib import MOE_ERR_UNSUPPORTED, MOE_OK, lib
from sparse_mixture_experts_gating_b200.workloads import (ACT_SWIGLU, DTYPE_BF16, GATE_RENORM, Workload,
                                                          make_inputs)

pytestmark = pytest.mark.gpu

W = Workload("no_alloc", T=150, d=512, E=8, k=2, d_ff=1024, act=ACT_SWIGLU, gate=GATE_RENORM,
             capacity_factor=1.0, dtype=DTYPE_BF16, bias="normal", seed=321)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _static_call(layer, inp, T):
    dev = inp["x"].device
    y = torch.full((T, layer.d), float("nan"), dtype=torch.bfloat16, device=dev)
    counts = torch.full((layer.E,), -1, dtype=torch.int32, device=dev)
    dropped = torch.full((1,), -1, dtype=torch.int32, device=dev)
    aux = torch.full((1,), float("nan"), device=dev)
    z = torch.full((1,), float("nan"), device=dev)
    rc = lib().moe_forward_static(layer._h, T, _p(inp["x"]), _p(inp["W_r"]), _p(inp["b_r"]), _p(inp["W1"]),
                                  _p(inp["W3"]), _p(inp["W2"]), _p(y), _p(counts), _p(dropped), _p(aux), _p(z),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, y, counts, dropped, aux, z


def test_static_scratch_entry_matches_moe_forward_on_two_calls_in_a_row():
    layer = MoELayer(W.E, W.k, W.d, W.d_ff, act=W.act, gate_mode=W.gate, capacity_factor=W.capacity_factor,
                     dtype=torch.bfloat16)
    assert layer.workspace_bytes(W.T) <= 32 << 20
    for seed in (321, 654):  # two calls in a row on the shared scratch, different inputs
        inp = make_inputs(W.with_(seed=seed), device="cuda")
        rc, y, counts, dropped, aux, z = _static_call(layer, inp, W.T)
        assert rc == MOE_OK, lib().moe_last_error().decode()
        status()
        y_ref, c_ref, d_ref, a_ref, z_ref = layer(inp["x"], inp["W_r"], inp["b_r"], inp["W1"], inp["W3"],
                                                  inp["W2"])
        status()
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
        assert torch.equal(counts, c_ref) and torch.equal(dropped, d_ref)
        assert torch.equal(aux.view(torch.int32), a_ref.view(torch.int32))
        assert torch.equal(z.view(torch.int32), z_ref.view(torch.int32))


def test_static_scratch_entry_rejects_a_layer_too_large_for_it():
    layer = MoELayer(8, 2, 4096, 14336, act="swiglu", gate_mode="renorm", dtype=torch.bfloat16)
    T = 1024
    assert layer.workspace_bytes(T) > 32 << 20
    x = torch.zeros((T, 4096), dtype=torch.bfloat16, device="cuda")
    inp = {"x": x, "W_r": torch.zeros((8, 4096), device="cuda"), "b_r": None, "W1": x, "W3": x, "W2": x}
    rc, y, counts, *_ = _static_call(layer, inp, T)
    assert rc == MOE_ERR_UNSUPPORTED
    assert "static scratch" in lib().moe_last_error().decode()
    torch.cuda.synchronize()
    assert torch.isnan(y.float()).all() and (counts == -1).all()
