"""The C++ loop oracle against the NumPy oracle (both pinned separately by
tests/test_oracle_pins.py): the same results on the same inputs, routing bit
for bit, floats to float64 rounding, whatever the thread count."""
import numpy as np
import pytest
import torch

import oracle
from oracle import cpp as oracle_cpp
from sparse_mixture_experts_gating_b200.workloads import (ACT_RELU, ACT_SWIGLU, DTYPE_BF16, GATE_RENORM,
                                                          GATE_SWITCH, Workload, make_inputs)

CPP = oracle_cpp.load()
rng = np.random.default_rng(11)

INT_KEYS = ("idx", "counts", "kept_counts", "offsets", "rank", "kept", "dest_row")
FLOAT_KEYS = ("p", "lse", "gate", "y")
SCALARS = ("dropped", "capacity", "aux", "z", "aux_all_choices", "cv_counts", "cv2_probs")


def _compare(a, b, rtol=1e-12):
    np.testing.assert_array_equal(a["logits"], b["logits"])
    for key in INT_KEYS:
        np.testing.assert_array_equal(a[key], b[key], err_msg=key)
    for key in FLOAT_KEYS:
        np.testing.assert_allclose(a[key], b[key], rtol=rtol, atol=rtol * max(1.0, np.abs(b[key]).max(initial=0)),
                                   err_msg=key)
    for key in SCALARS:
        if isinstance(b[key], float):
            assert a[key] == pytest.approx(b[key], rel=rtol, abs=rtol), key
        else:
            assert a[key] == b[key], key


@pytest.mark.parametrize("act", [ACT_RELU, ACT_SWIGLU])
@pytest.mark.parametrize("gate", [GATE_SWITCH, GATE_RENORM])
@pytest.mark.parametrize("T,d,E,k,d_ff,cf,ns", [(50, 16, 6, 2, 24, 0.8, 0), (97, 12, 8, 3, 20, 0.0, 1),
                                                  (40, 8, 1, 1, 10, 1.0, 0), (64, 10, 5, 5, 7, 0.0, 2),
                                                  (0, 8, 4, 2, 8, 1.0, 0)])
def test_cpp_and_numpy_oracles_agree_on_float64_layers(act, gate, T, d, E, k, d_ff, cf, ns):
    x = rng.normal(size=(T, d)); W_r = rng.normal(size=(E, d)); b = rng.normal(size=E)
    W1 = rng.normal(size=(E + ns, d_ff, d)); W3 = rng.normal(size=(E + ns, d_ff, d))
    W2 = rng.normal(size=(E + ns, d, d_ff))
    shared = None if not ns else (W1[E:], W3[E:] if act else None, W2[E:])
    kw = dict(k=k, gate_mode=gate, act=act, capacity_factor=cf, shared=shared)
    a = CPP.moe_forward(x, W_r, b, W1, W3 if act else None, W2, **kw)
    b_ = oracle.moe_forward(x, W_r, b, W1, W3 if act else None, W2, **kw)
    _compare(a, b_)


def test_bf16_weights_are_read_as_their_exact_values():
    """bf16 tensors go to the C++ oracle as bit patterns, to NumPy as float32
    copies: the same numbers, so the same results."""
    w = Workload("bf16_mix", T=300, d=64, E=8, k=2, d_ff=96, act=ACT_SWIGLU, gate=GATE_RENORM, capacity_factor=1.0,
                 dtype=DTYPE_BF16, bias="normal", dyadic=True, seed=5, n_shared=1)
    inp = make_inputs(w)
    h = {key: (None if v is None else v.float().numpy()) for key, v in inp.items()}
    shared_t = (inp["W1"][w.E:], inp["W3"][w.E:], inp["W2"][w.E:])
    shared_h = (h["W1"][w.E:], h["W3"][w.E:], h["W2"][w.E:])
    kw = dict(k=w.k, gate_mode=w.gate, act=w.act, capacity_factor=w.capacity_factor)
    a = CPP.moe_forward(inp["x"], inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"], shared=shared_t, **kw)
    b = oracle.moe_forward(h["x"], h["W_r"], h["b_r"], h["W1"][:w.E], h["W3"][:w.E], h["W2"][:w.E],
                           shared=shared_h, **kw)
    assert a["dropped"] > 0
    _compare(a, b)


def test_results_do_not_depend_on_threads_or_on_the_rows_asked_for():
    T, d, E, k, d_ff = 120, 16, 6, 2, 32
    x = rng.normal(size=(T, d)); W_r = rng.normal(size=(E, d))
    W1 = rng.normal(size=(E, d_ff, d)); W3 = rng.normal(size=(E, d_ff, d)); W2 = rng.normal(size=(E, d, d_ff))
    kw = dict(k=k, gate_mode=GATE_RENORM, act=ACT_SWIGLU, capacity_factor=0.9)
    one = CPP.moe_forward(x, W_r, None, W1, W3, W2, threads=1, **kw)
    many = CPP.moe_forward(x, W_r, None, W1, W3, W2, threads=7, **kw)
    rows = [119, 3, 64, 0]
    part = CPP.moe_forward(x, W_r, None, W1, W3, W2, rows=rows, threads=3, **kw)
    for key in INT_KEYS + FLOAT_KEYS:
        np.testing.assert_array_equal(one[key], many[key], err_msg=key)
    np.testing.assert_array_equal(part["y"], one["y"][rows])


def test_given_logits_route_both_oracles_identically():
    T, E, k = 200, 16, 4
    logits = (rng.integers(-8, 8, size=(T, E)) / 4).astype(np.float32)  # many ties
    x = np.zeros((T, 4)); W = np.zeros((E, 4))
    z1, z2 = np.zeros((E, 3, 4)), np.zeros((E, 4, 3))
    kw = dict(k=k, gate_mode=GATE_RENORM, act=ACT_RELU, capacity_factor=1.0, logits=logits)
    _compare(CPP.moe_forward(x, W, None, z1, None, z2, **kw), oracle.moe_forward(x, W, None, z1, None, z2, **kw))


def test_torch_float32_and_float64_inputs():
    T, d, E = 30, 8, 4
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(3))
    W_r = torch.randn(E, d, generator=torch.Generator().manual_seed(4))
    W1 = torch.randn(E, 12, d, dtype=torch.float64, generator=torch.Generator().manual_seed(5))
    W2 = torch.randn(E, d, 12, dtype=torch.float64, generator=torch.Generator().manual_seed(6))
    kw = dict(k=2, gate_mode=GATE_SWITCH, act=ACT_RELU, capacity_factor=0.0)
    a = CPP.moe_forward(x, W_r, None, W1, None, W2, **kw)
    b = oracle.moe_forward(x.numpy(), W_r.numpy(), None, W1.numpy(), None, W2.numpy(), **kw)
    _compare(a, b)
