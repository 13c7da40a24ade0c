"""CPU oracle for the backward pass of the sparse Mixture-of-Experts layer.

TEST INFRASTRUCTURE ONLY (see moe_oracle.py): only tests/,
``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg may import or run
it; the product path never does.

Gradients of the scalar

    L = sum_t <dy_t, y_t> + aux_coef * aux + z_coef * z

with respect to x, W_r, b_r and the expert weights, for the layer of
moe_oracle.moe_forward, in float64.  What the pages fix:

  * "Mixture of experts" (rayaq.ca), section "Replacing the feed-forward
    block": the choice of experts is discrete and the router learns only
    through the gate values that multiply each expert's output.  So the top-k
    selection and the capacity drops are held fixed (no gradient), and a
    dropped assignment, which adds nothing to y, passes no gradient.
  * same page, section "The load-balancing loss": f_i is a count and has no
    gradient; P_i (the mean full-softmax probability) does, with
    d(f_i P_i)/dP_i = f_i.  The z-loss is the mean over tokens of lse^2, so
    dz/dh_te = (2 / T) lse_t p_te.
  * gates ("Top-k gating"): Switch g = p_idx (full softmax); renormalised g =
    softmax over the k chosen logits.

Readings where the pages are silent (listed in the design notes):
  - the gradient is the exact derivative of the forward with routing held
    fixed (no straight-through estimate through the selection);
  - the rounding of the router logits to float32 passes the gradient as the
    identity;
  - the alternative balance statistics are reported, not differentiated.

Pins: tests/test_oracle_backward.py checks every gradient against central
finite differences of moe_oracle.moe_forward (float64 logits) on small
layers whose routing, drops and ReLU signs do not change under the step,
plus the closed form of the one-expert router gradient.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from .moe_oracle import (ACT_RELU, GATE_SWITCH, assign_slots, expert_capacity, gates, router_logits,
                         softmax_lse, top_k)


def _expert_backward(xr, W1e, W3e, W2e, act: int, dout):
    """Backward of one expert FFN on a batch of rows ("Implementation":
    w2(silu(w1 x) * w3 x); ReLU: w2(relu(w1 x))).

    xr [n][d], dout [n][d] (the gradient reaching the expert's output rows).
    Returns (out [n][d], dx [n][d], dW1 [d_ff][d], dW3 or None, dW2 [d][d_ff]).
    silu'(u) = s + u s (1 - s) with s the logistic function.
    """
    W1e = np.asarray(W1e, np.float64)
    W2e = np.asarray(W2e, np.float64)
    a1 = xr @ W1e.T
    if act == ACT_RELU:
        hdn = np.maximum(a1, 0.0)
    else:
        W3e = np.asarray(W3e, np.float64)
        a3 = xr @ W3e.T
        s = 1.0 / (1.0 + np.exp(-a1))
        silu = a1 * s
        hdn = silu * a3
    out = hdn @ W2e.T
    dW2 = dout.T @ hdn
    dh = dout @ W2e
    if act == ACT_RELU:
        da1 = dh * (a1 > 0.0)
        dx = da1 @ W1e
        return out, dx, da1.T @ xr, None, dW2
    da3 = dh * silu
    da1 = dh * a3 * (s + a1 * s * (1.0 - s))
    dx = da1 @ W1e + da3 @ W3e
    return out, dx, da1.T @ xr, da3.T @ xr, dW2


def _router_backward(p, lse, idx, g, dg, gate_mode: int, aux_coef: float, z_coef: float):
    """Gradient reaching the router logits h [T][E] from the gate gradients dg
    [T][k], the load-balancing loss and the z-loss ("Top-k gating" and "The
    load-balancing loss").

    Switch: g_j = p[idx_j], so dg flows into dp and through the softmax.
    Renormalised: g = softmax over the chosen logits, so
    dh_{idx_j} = g_j (dg_j - sum_i g_i dg_i) and the other logits get nothing.
    aux = E sum_i f_i P_i with f constant: dp_ti += aux_coef E f_i / T.
    Softmax: dh = p * (dp - <dp, p>).  z = mean_t lse_t^2: dh += z_coef (2/T) lse_t p.
    """
    T, E = p.shape
    rows = np.broadcast_to(np.arange(T)[:, None], idx.shape)
    dh = np.zeros((T, E))
    dp = np.zeros((T, E))
    if gate_mode == GATE_SWITCH:
        np.add.at(dp, (rows, idx), dg)
    else:
        np.add.at(dh, (rows, idx), g * (dg - np.sum(g * dg, axis=1, keepdims=True)))
    if T > 0:
        f = np.bincount(idx[:, 0], minlength=E).astype(np.float64) / T  # a count: constant
        dp += aux_coef * E * f[None, :] / T
    dh += p * (dp - np.sum(dp * p, axis=1, keepdims=True))
    if T > 0:
        dh += z_coef * (2.0 / T) * lse[:, None] * p
    return dh


def moe_backward(x, W_r, b_r, W1, W3, W2, dy, *, k: int, gate_mode: int, act: int, capacity_factor: float,
                 aux_coef: float = 0.0, z_coef: float = 0.0, shared: Optional[tuple] = None,
                 logits_dtype=np.float32) -> dict:
    """Gradients of L = <dy, y> + aux_coef * aux + z_coef * z (see the module
    docstring).  Arguments as moe_oracle.moe_forward; dy [T][d].

    Returns dx [T][d], dW_r [E][d], db_r [E], dW1 / dW3 [E][d_ff][d] (dW3 None
    for ReLU), dW2 [E][d][d_ff], dg [T][k] (the gradient reaching each gate,
    0 where dropped), dh [T][E] (the gradient reaching the logits), and for
    shared experts dW1s / dW3s / dW2s.
    """
    x = np.asarray(x, np.float64)
    dy = np.asarray(dy, np.float64)
    T, d = x.shape
    E = np.asarray(W_r).shape[0]
    h = router_logits(x, W_r, b_r, logits_dtype)
    p, lse = softmax_lse(h)
    idx = top_k(h, k)
    g = gates(h, p, idx, gate_mode)
    slots = assign_slots(idx, E, expert_capacity(capacity_factor, T, k, E))
    kept = slots["kept"]

    dx = np.zeros((T, d))
    dW1 = np.zeros(np.shape(W1))
    dW3 = None if W3 is None else np.zeros(np.shape(W3))
    dW2 = np.zeros(np.shape(W2))
    dg = np.zeros((T, k))
    for e in range(E):
        ts, js = np.nonzero((idx == e) & kept)
        if ts.size == 0:
            continue
        ge = g[ts, js][:, None]
        out, dxe, d1, d3, d2 = _expert_backward(x[ts], W1[e], None if W3 is None else W3[e], W2[e], act,
                                                ge * dy[ts])
        dg[ts, js] = np.sum(dy[ts] * out, axis=1)
        np.add.at(dx, ts, dxe)
        dW1[e] += d1
        if dW3 is not None:
            dW3[e] += d3
        dW2[e] += d2

    res = {}
    if shared is not None:
        W1s, W3s, W2s = shared
        res["dW1s"] = np.zeros(np.shape(W1s))
        res["dW3s"] = None if W3s is None else np.zeros(np.shape(W3s))
        res["dW2s"] = np.zeros(np.shape(W2s))
        for si in range(len(W1s)):
            _, dxs, d1, d3, d2 = _expert_backward(x, W1s[si], None if W3s is None else W3s[si], W2s[si], act, dy)
            dx += dxs
            res["dW1s"][si] = d1
            if d3 is not None:
                res["dW3s"][si] = d3
            res["dW2s"][si] = d2

    dh = _router_backward(p, lse, idx, g, dg, gate_mode, aux_coef, z_coef)
    dx += dh @ np.asarray(W_r, np.float64)
    res.update({
        "dx": dx, "dW_r": dh.T @ x, "db_r": dh.sum(axis=0), "dW1": dW1, "dW3": dW3, "dW2": dW2,
        "dg": dg, "dh": dh, "idx": idx, "kept": kept,
    })
    return res


def loss_value(x, W_r, b_r, W1, W3, W2, dy, *, k: int, gate_mode: int, act: int, capacity_factor: float,
               aux_coef: float = 0.0, z_coef: float = 0.0, shared: Optional[tuple] = None,
               logits_dtype=np.float32):
    """L = sum_t <dy_t, y_t> + aux_coef * aux + z_coef * z from the forward
    oracle, with its routing (idx, kept) for checking that a finite-difference
    step left the routing alone."""
    from .moe_oracle import moe_forward
    f = moe_forward(x, W_r, b_r, W1, W3, W2, k=k, gate_mode=gate_mode, act=act, capacity_factor=capacity_factor,
                    shared=shared, logits_dtype=logits_dtype)
    L = float(np.sum(np.asarray(dy, np.float64) * f["y"])) + aux_coef * f["aux"] + z_coef * f["z"]
    return L, f["idx"], f["kept"]
