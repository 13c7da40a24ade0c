"""Pins of the backward oracle (oracle/moe_backward.py), CPU only.

Every gradient is checked against central finite differences of the forward
oracle's loss L = <dy, y> + aux_coef * aux + z_coef * z, computed with
float64 logits (a float32 rounding would swamp the steps), on small layers
whose routing, capacity drops and ReLU signs stay the same across every step
(checked per step).  The finite differences know nothing of the backward
formulas: a dropped term, a wrong sign or a transposed operand anywhere in the
backward shows up as a mismatch.  Plus the closed form of the one-expert case,
where only the z-loss reaches the router: dL/dh_t = z_coef * 2 h_t / T.
"""
import numpy as np
import pytest

import oracle
from oracle import moe_backward as B

F64 = np.float64
EPS = 1e-5


def _layer(seed, T, d, E, k, d_ff, act, gate, cf, bias, n_shared=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    W_r = rng.standard_normal((E, d)) / np.sqrt(d)
    b_r = rng.standard_normal(E) * 0.5 if bias else None
    W1 = rng.standard_normal((E, d_ff, d)) / np.sqrt(d)
    W3 = rng.standard_normal((E, d_ff, d)) / np.sqrt(d) if act == oracle.ACT_SWIGLU else None
    W2 = rng.standard_normal((E, d, d_ff)) / np.sqrt(d_ff)
    shared = None
    if n_shared:
        shared = (rng.standard_normal((n_shared, d_ff, d)) / np.sqrt(d),
                  rng.standard_normal((n_shared, d_ff, d)) / np.sqrt(d) if act == oracle.ACT_SWIGLU else None,
                  rng.standard_normal((n_shared, d, d_ff)) / np.sqrt(d_ff))
    dy = rng.standard_normal((T, d))
    return dict(x=x, W_r=W_r, b_r=b_r, W1=W1, W3=W3, W2=W2, dy=dy, shared=shared,
                kw=dict(k=k, gate_mode=gate, act=act, capacity_factor=cf))


CASES = {
    # Switch k = 1, ReLU, capacity drops, bias
    "switch_relu_drops": (11, 9, 5, 4, 1, 6, oracle.ACT_RELU, oracle.GATE_SWITCH, 1.0, True, 0),
    # renormalised top-2, SwiGLU, dropless
    "renorm_swiglu_k2": (12, 7, 4, 5, 2, 6, oracle.ACT_SWIGLU, oracle.GATE_RENORM, 0.0, False, 0),
    # Switch gates with k = 2 (each gate a full-softmax probability), SwiGLU, drops
    "switch_k2_swiglu_drops": (13, 8, 4, 4, 2, 5, oracle.ACT_SWIGLU, oracle.GATE_SWITCH, 0.75, True, 0),
    # a shared expert beside renormalised top-2 ReLU experts
    "shared_relu": (14, 6, 4, 4, 2, 5, oracle.ACT_RELU, oracle.GATE_RENORM, 0.0, True, 1),
}
COEF = dict(aux_coef=0.37, z_coef=0.21)


def _loss(L, **over):
    p = dict(L, **over)
    return B.loss_value(p["x"], p["W_r"], p["b_r"], p["W1"], p["W3"], p["W2"], p["dy"], shared=p["shared"],
                        logits_dtype=F64, **p["kw"], **COEF)


_SHARED = {"W1s": 0, "W3s": 1, "W2s": 2}


def _get(L, name):
    return L["shared"][_SHARED[name]] if name in _SHARED else L[name]


def _with(L, name, arr):
    if name in _SHARED:
        sh = list(L["shared"])
        sh[_SHARED[name]] = arr
        return {"shared": tuple(sh)}
    return {name: arr}


def _fd(L, name, grad):
    """Worst relative mismatch of central differences over every entry of `name`."""
    base = _get(L, name)
    _, idx0, kept0 = _loss(L)
    worst = 0.0
    for pos in np.ndindex(*base.shape):
        vals = []
        for s in (+1, -1):
            arr = base.copy()
            arr[pos] += s * EPS
            v, idx, kept = _loss(L, **_with(L, name, arr))
            assert np.array_equal(idx, idx0) and np.array_equal(kept, kept0), "routing moved under the step"
            vals.append(v)
        num = (vals[0] - vals[1]) / (2 * EPS)
        worst = max(worst, abs(num - grad[pos]) / (1.0 + abs(grad[pos])))
    return worst


def _relu_margin(L):
    """Smallest |w1 x| over every expert and token (ReLU kinks stay away from the steps)."""
    a = np.einsum("td,efd->tef", L["x"], L["W1"])
    m = np.abs(a).min()
    if L["shared"] is not None:
        m = min(m, np.abs(np.einsum("td,sfd->tsf", L["x"], L["shared"][0])).min())
    return m


@pytest.mark.parametrize("case", sorted(CASES))
def test_gradients_match_finite_differences(case):
    seed, *shape = CASES[case]

    def usable(L):  # ReLU inputs off the kink; a case with a capacity drops something
        if L["kw"]["act"] == oracle.ACT_RELU and _relu_margin(L) <= 1e-3:
            return False
        return L["kw"]["capacity_factor"] <= 0 or not _loss(L)[2].all()

    L = next(L for L in (_layer(s, *shape) for s in range(seed, seed + 5000, 97)) if usable(L))
    g = B.moe_backward(L["x"], L["W_r"], L["b_r"], L["W1"], L["W3"], L["W2"], L["dy"], shared=L["shared"],
                       logits_dtype=F64, **L["kw"], **COEF)
    assert g["kept"].sum() > 0
    if L["kw"]["capacity_factor"] > 0:
        assert not g["kept"].all(), "the case should drop some assignments"
    checks = {"x": g["dx"], "W_r": g["dW_r"], "W1": g["dW1"], "W2": g["dW2"]}
    if L["b_r"] is not None:
        checks["b_r"] = g["db_r"]
    if L["W3"] is not None:
        checks["W3"] = g["dW3"]
    for name, grad in checks.items():
        assert _fd(L, name, grad) < 1e-7, name
    if L["shared"] is not None:
        for name, key in (("W1s", "dW1s"), ("W2s", "dW2s")):
            assert _fd(L, name, g[key]) < 1e-7, name


def test_one_expert_router_gradient_closed_form():
    """E = 1: p = 1 and the gate is 1 whatever the logit, so dy and the
    load-balancing loss pass nothing to the router; the z-loss (1/T) sum h_t^2
    gives dL/dh_t = z_coef * 2 h_t / T, hence dW_r = sum_t that * x_t."""
    L = _layer(21, 6, 4, 1, 1, 5, oracle.ACT_RELU, oracle.GATE_SWITCH, 0.0, True)
    g = B.moe_backward(L["x"], L["W_r"], L["b_r"], L["W1"], L["W3"], L["W2"], L["dy"], logits_dtype=F64,
                       aux_coef=0.5, z_coef=0.3, **L["kw"])
    h = L["x"] @ L["W_r"][0] + L["b_r"][0]
    dh = 0.3 * 2.0 * h / 6
    np.testing.assert_allclose(g["dh"][:, 0], dh, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(g["dW_r"][0], dh @ L["x"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(g["db_r"][0], dh.sum(), rtol=1e-12, atol=1e-14)


def test_gradients_are_linear_in_dy_and_zero_without_loss():
    L = _layer(22, 7, 4, 4, 2, 5, oracle.ACT_SWIGLU, oracle.GATE_RENORM, 1.0, True)
    kw = dict(shared=None, **L["kw"])
    g0 = B.moe_backward(L["x"], L["W_r"], L["b_r"], L["W1"], L["W3"], L["W2"], 0 * L["dy"], **kw)
    for key in ("dx", "dW_r", "dW1", "dW3", "dW2"):
        assert not np.any(g0[key]), key
    g1 = B.moe_backward(L["x"], L["W_r"], L["b_r"], L["W1"], L["W3"], L["W2"], L["dy"], **kw)
    g3 = B.moe_backward(L["x"], L["W_r"], L["b_r"], L["W1"], L["W3"], L["W2"], 3 * L["dy"], **kw)
    for key in ("dx", "dW_r", "dW1", "dW3", "dW2"):
        np.testing.assert_allclose(g3[key], 3 * g1[key], rtol=1e-12, atol=1e-12)


def test_dropped_assignments_pass_no_gradient():
    """A token whose every assignment is dropped reaches no expert weight and
    gets no expert part of dx: its dx is the router part alone."""
    L = _layer(23, 10, 4, 4, 1, 5, oracle.ACT_RELU, oracle.GATE_SWITCH, 0.3, False)
    g = B.moe_backward(L["x"], L["W_r"], L["b_r"], L["W1"], L["W3"], L["W2"], L["dy"], **L["kw"])
    dropped = np.nonzero(~g["kept"][:, 0])[0]
    assert dropped.size > 0
    np.testing.assert_allclose(g["dx"][dropped], (g["dh"] @ L["W_r"])[dropped], rtol=1e-12, atol=1e-14)
    assert not np.any(g["dg"][dropped])


# --------------------------------------------------------------------------
# Planted mistakes: each must fail the finite-difference pin of some case.

def _silu_grad_without_second_term(xr, W1e, W3e, W2e, act, dout):
    out, dx, d1, d3, d2 = _orig_expert(xr, W1e, W3e, W2e, act, dout)
    if act == oracle.ACT_RELU:
        return out, dx, d1, d3, d2
    a1 = xr @ np.asarray(W1e).T
    a3 = xr @ np.asarray(W3e).T
    s = 1 / (1 + np.exp(-a1))
    da1 = (dout @ np.asarray(W2e)) * a3 * s
    return out, da1 @ W1e + (dx - ((dout @ np.asarray(W2e)) * a3 * (s + a1 * s * (1 - s))) @ W1e), da1.T @ xr, d3, d2


def _dx_without_w3(xr, W1e, W3e, W2e, act, dout):
    out, dx, d1, d3, d2 = _orig_expert(xr, W1e, W3e, W2e, act, dout)
    if act == oracle.ACT_RELU:
        return out, dx, d1, d3, d2
    da3 = (dout @ np.asarray(W2e)) * (xr @ np.asarray(W1e).T) / (1 + np.exp(-(xr @ np.asarray(W1e).T)))
    return out, dx - da3 @ W3e, d1, d3, d2


def _softmax_not_centred(p, lse, idx, g, dg, gate_mode, aux_coef, z_coef):
    dh = _orig_router(p, lse, idx, g, dg, gate_mode, aux_coef, z_coef)
    T, E = p.shape
    dp = np.zeros((T, E))
    if gate_mode == oracle.GATE_SWITCH:
        np.add.at(dp, (np.broadcast_to(np.arange(T)[:, None], idx.shape), idx), dg)
    return dh + p * np.sum(dp * p, axis=1, keepdims=True)


def _aux_grad_missing_T(p, lse, idx, g, dg, gate_mode, aux_coef, z_coef):
    return _orig_router(p, lse, idx, g, dg, gate_mode, aux_coef * p.shape[0], z_coef)


def _renorm_gate_grad_uncentred(p, lse, idx, g, dg, gate_mode, aux_coef, z_coef):
    dh = _orig_router(p, lse, idx, g, dg, gate_mode, aux_coef, z_coef)
    if gate_mode == oracle.GATE_SWITCH:
        return dh
    rows = np.broadcast_to(np.arange(p.shape[0])[:, None], idx.shape)
    np.add.at(dh, (rows, idx), g * np.sum(g * dg, axis=1, keepdims=True))
    return dh


def _z_grad_sign(p, lse, idx, g, dg, gate_mode, aux_coef, z_coef):
    return _orig_router(p, lse, idx, g, dg, gate_mode, aux_coef, -z_coef)


_orig_expert = B._expert_backward
_orig_router = B._router_backward
BW_MUTANTS = {
    "silu_grad_without_second_term": ("_expert_backward", _silu_grad_without_second_term),
    "dx_without_w3": ("_expert_backward", _dx_without_w3),
    "softmax_not_centred": ("_router_backward", _softmax_not_centred),
    "aux_grad_missing_T": ("_router_backward", _aux_grad_missing_T),
    "renorm_gate_grad_uncentred": ("_router_backward", _renorm_gate_grad_uncentred),
    "z_grad_sign": ("_router_backward", _z_grad_sign),
}


@pytest.mark.parametrize("name", sorted(BW_MUTANTS))
def test_backward_mutant_is_caught(name, monkeypatch):
    attr, fn = BW_MUTANTS[name]
    monkeypatch.setattr(B, attr, fn)
    caught = False
    for case in sorted(CASES):
        try:
            test_gradients_match_finite_differences(case)
        except AssertionError:
            caught = True
            break
    assert caught, name
