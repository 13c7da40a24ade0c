"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare them.

Tolerances (derived from the arithmetic; see the design notes):
  * routing (top-k indices, expert counts, offsets, destination rows, drop
    mask, dropped count): bit-exact;
  * fp32 layers: max|dy| / max|y_ref| <= 1e-5;
  * bf16 layers, always against the plain oracle (float64, nothing rounded
    between its steps): max|dy| <= 1e-2 * RMS(y_ref) on the fp32-accumulated
    value of y before its final cast, and sum|dy| / sum|y_ref| <= 2e-3 both on
    that value and on the returned bf16 y; the returned y must be exactly the
    round-to-nearest-even image of the fp32 value.  With the hidden activation
    held in ONE bf16 plane (MOE_HIDDEN_BF16) its rounding alone (unit roundoff
    2^-8) pushes the max to ~1.5e-2 * RMS on large outputs and adds ~1.6e-3 of
    mean relative error, on top of the ~1.3e-3 of the final cast: that mode is
    outside the bar; it is held to the mean bound on the fp32 value and to
    3e-3 (the sum of the two terms) on the returned bf16 y, its max error is
    reported;
  * gates: |dg| <= 2e-6 (fp32 exp of exact logit differences);
  * aux, z: relative 1e-5.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from sparse_mixture_experts_gating_b200 import MoELayer, status
from sparse_mixture_experts_gating_b200.workloads import DTYPE_F32, Workload, make_inputs, torch_dtype


def np32(t):
    return None if t is None else t.detach().float().cpu().numpy()


class HostExperts:
    """Per-expert host copies of a device weight [E][rows][cols] (fp32 numpy)."""

    def __init__(self, t):
        self.t = t
        self.cache = {}

    def __getitem__(self, e):
        if e not in self.cache:
            self.cache[e] = self.t[e].float().cpu().numpy()
        return self.cache[e]


def layer_for(w: Workload, hidden: str = "auto") -> MoELayer:
    return MoELayer(w.E, w.k, w.d, w.d_ff, act=w.act, gate_mode=w.gate,
                    capacity_factor=w.capacity_factor, dtype=torch_dtype(w.dtype), hidden=hidden,
                    n_shared=w.n_shared)


def run_gpu(w: Workload, inp: dict, *, logits_in=None, debug=True, layer=None):
    layer = layer or layer_for(w)
    dev = inp["x"].device
    dbg = layer.debug_buffers(w.T, dev) if debug else None
    if logits_in is not None:
        dbg = dbg or {}
        dbg["logits_in"] = logits_in
    y, counts, dropped, aux, z = layer(inp["x"], inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"],
                                       debug=dbg)
    status()
    out = {"y_dev": y, "y": np32(y), "counts": counts.cpu().numpy(), "dropped": int(dropped.item()),
           "aux": float(aux.item()), "z": float(z.item())}
    bl = layer.balance_losses(w.T).cpu().numpy()
    out.update(aux_all_choices=float(bl[0]), cv_counts=float(bl[1]), cv2_probs=float(bl[2]))
    if dbg:
        for key, t in dbg.items():
            if key != "logits_in":
                out[key] = t.cpu().numpy() if t.dtype != torch.float32 else np32(t)
        out["y_f32_dev"] = dbg.get("y_f32")
    return out


def host_inputs(inp: dict):
    return {"x": np32(inp["x"]), "W_r": np32(inp["W_r"]), "b_r": np32(inp["b_r"]),
            "W1": HostExperts(inp["W1"]), "W3": None if inp["W3"] is None else HostExperts(inp["W3"]),
            "W2": HostExperts(inp["W2"])}


class _Shift:
    """Experts E + s of a HostExperts as a sequence of n shared experts."""

    def __init__(self, he, E, n):
        self.he, self.E, self.n = he, E, n

    def __len__(self):
        return self.n

    def __getitem__(self, s):
        return self.he[self.E + s]


def run_oracle(w: Workload, host: dict, rows=None, logits=None):
    shared = None
    if w.n_shared:
        shared = (_Shift(host["W1"], w.E, w.n_shared),
                  None if host["W3"] is None else _Shift(host["W3"], w.E, w.n_shared),
                  _Shift(host["W2"], w.E, w.n_shared))
    return O.moe_forward(host["x"], host["W_r"], host["b_r"], host["W1"], host["W3"], host["W2"],
                         k=w.k, gate_mode=w.gate, act=w.act, capacity_factor=w.capacity_factor,
                         rows=rows, logits=logits, shared=shared)


def assert_routing_equal(g: dict, o: dict):
    np.testing.assert_array_equal(g["topk_idx"], o["idx"])
    np.testing.assert_array_equal(g["counts"], o["counts"])
    np.testing.assert_array_equal(g["expert_offsets"], o["offsets"])
    np.testing.assert_array_equal(g["dest_row"], o["dest_row"])
    np.testing.assert_array_equal(g["drop_mask"].astype(bool), ~o["kept"])
    assert g["dropped"] == o["dropped"]


def assert_gates_and_losses(g: dict, o: dict):
    np.testing.assert_allclose(g["topk_gate"], o["gate"], rtol=0, atol=2e-6)
    assert abs(g["aux"] - o["aux"]) <= 1e-5 * max(1.0, abs(o["aux"]))
    assert abs(g["z"] - o["z"]) <= 1e-5 * max(1.0, abs(o["z"]))
    # the alternative balance statistics (fp32 results of fp64 sums of fp32 partials)
    for key in ("aux_all_choices", "cv_counts", "cv2_probs"):
        if key in g:
            assert abs(g[key] - o[key]) <= 1e-5 * max(1.0, abs(o[key])), (key, g[key], o[key])
    if "lse_out" in g:
        np.testing.assert_allclose(g["lse_out"], o["lse"], rtol=2e-6, atol=2e-6)


def y_errors(y_gpu: np.ndarray, y_ref: np.ndarray):
    d = np.abs(y_gpu.astype(np.float64) - y_ref)
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    return {
        "max_abs": float(d.max()) if d.size else 0.0,
        "rms_ref": rms,
        "max_over_rms": float(d.max() / rms) if d.size and rms > 0 else 0.0,
        "max_rel_to_max": float(d.max() / np.abs(y_ref).max()) if d.size and np.abs(y_ref).max() > 0 else 0.0,
        "mean_rel": float(d.sum() / np.abs(y_ref).sum()) if d.size and np.abs(y_ref).sum() > 0 else 0.0,
    }


def assert_y_close(w: Workload, g: dict, y_ref: np.ndarray, rows=None, single_plane_hidden=False):
    """y of the CUDA path against the plain oracle y_ref.

    fp32 layers: max|dy| / max|y_ref| <= 1e-5.  bf16 layers: the mean bound
    2e-3 on the fp32 value before the cast and on the returned bf16 y, the max
    bound 1e-2 * RMS(y_ref) on the fp32 value, and the returned y bit for bit
    the round-to-nearest-even image of the fp32 value.  single_plane_hidden
    (the MOE_HIDDEN_BF16 mode, outside the bar): no max bound, and 3e-3 for
    the mean of the returned bf16 y.
    """
    sel = slice(None) if rows is None else np.asarray(rows)
    if w.dtype == DTYPE_F32:
        e = y_errors(g["y"][sel], y_ref)
        assert e["max_rel_to_max"] <= 1e-5, e
        return e
    yf = g["y_f32"][sel]
    e = y_errors(yf, y_ref)
    e["bf16_output"] = y_errors(g["y"][sel], y_ref)
    assert e["mean_rel"] <= 2e-3, e
    assert e["bf16_output"]["mean_rel"] <= (3e-3 if single_plane_hidden else 2e-3), e
    if not single_plane_hidden:
        assert e["max_over_rms"] <= 1e-2, e
    # the bf16 output is the RNE image of the fp32 value
    rne = torch.from_numpy(np.ascontiguousarray(yf)).to(torch.bfloat16)
    out = g["y_dev"].cpu()
    if rows is not None:
        out = out[torch.as_tensor(np.asarray(rows))]
    assert torch.equal(rne.view(torch.int16), out.view(torch.int16))
    return e


def sample_rows(w: Workload, o_or_kept=None, n=48, seed=0):
    rng = np.random.default_rng(seed)
    rows = {0, w.T - 1} | set(rng.integers(0, w.T, size=min(n, w.T)).tolist())
    if o_or_kept is not None:  # include some dropped / partially dropped tokens
        gone = np.nonzero(~o_or_kept.all(axis=1))[0]
        rows |= set(gone[:8].tolist()) | set(gone[-8:].tolist())
    return np.array(sorted(rows))


def make(w: Workload, device="cuda"):
    return make_inputs(w, device=device)
