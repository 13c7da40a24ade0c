"""Each plausible mistake planted in the oracle must fail at least one pin.

The mutants live only here, on the CPU.  For the NumPy oracle they patch the
module's functions for the duration of one check; for the C++ oracle they are
textual edits of a copy of oracle/moe_oracle.cpp, compiled into a temporary
library.  This shows the pins in test_oracle_pins.py would catch a dropped
term, a wrong sign, a wrong index or tie rule, a transposed operand, an
off-by-one capacity, a wrong slot priority, a wrong moment in the balance
statistics or shared experts applied to the wrong tokens or weights, in
either implementation.
"""
import numpy as np
import pytest

import oracle
import oracle.moe_oracle as M
from oracle import cpp as oracle_cpp
from tests import test_oracle_pins as P


def _top_k_last_index_on_ties(h32, k):
    h = np.asarray(h32, np.float64)[:, ::-1].copy()
    E = h.shape[1]
    idx = np.empty((h.shape[0], k), np.int64)
    rows = np.arange(h.shape[0])
    for j in range(k):
        s = np.argmax(h, axis=1)
        idx[:, j] = E - 1 - s
        h[rows, s] = -np.inf
    return idx


def _gates_not_renormalised(h32, p, idx, gate_mode):
    return p[np.arange(idx.shape[0])[:, None], idx]


def _ffn_silu_sign(xr, W1e, W3e, W2e, act):
    a = xr @ np.asarray(W1e, np.float64).T
    hdn = np.maximum(a, 0) if act == M.ACT_RELU else a / (1 + np.exp(a)) * (xr @ np.asarray(W3e, np.float64).T)
    return hdn @ np.asarray(W2e, np.float64).T


def _ffn_w1_w3_swapped_roles(xr, W1e, W3e, W2e, act):
    if act == M.ACT_RELU:
        return _orig["expert_ffn"](xr, W1e, W3e, W2e, act)
    a = xr @ np.asarray(W3e, np.float64).T
    b = xr @ np.asarray(W1e, np.float64).T
    return (a / (1 + np.exp(-a)) * b) @ np.asarray(W2e, np.float64).T


def _aux_without_E(p, lse, idx, E):
    aux, z = _orig["aux_and_z"](p, lse, idx, E)
    return aux / E, z


def _z_without_square(p, lse, idx, E):
    aux, _ = _orig["aux_and_z"](p, lse, idx, E)
    return aux, float(np.mean(lse)) if len(lse) else 0.0


def _f_over_all_choices(p, lse, idx, E):
    T = p.shape[0]
    f = np.bincount(idx.reshape(-1), minlength=E) / (T * idx.shape[1])
    return float(E * np.sum(f * p.mean(axis=0))), float(np.mean(lse ** 2))


def _slots_off_by_one(idx, E, C):
    return _orig["assign_slots"](idx, E, None if C is None else C + 1)


def _slots_choice_major(idx, E, C):
    T, k = idx.shape
    s = _orig["assign_slots"](idx.T.copy(), E, C)  # scans choice j before token t
    for key in ("rank", "kept", "dest_row"):
        s[key] = s[key].T.copy()
    return s


def _logits_transposed_router(x, W_r, b_r=None, dtype=np.float32):
    W = np.asarray(W_r, np.float64)
    h = np.asarray(x, np.float64) @ (W.T if W.shape[0] != W.shape[1] else W)
    if b_r is not None:
        h = h + b_r
    return h.astype(dtype)


def _logits_dropped_bias(x, W_r, b_r=None, dtype=np.float32):
    return _orig["router_logits"](x, W_r, None, dtype)


def _balance_sample_std(p, idx, E):
    r = _orig["balance_losses"](p, idx, E)
    counts = np.bincount(idx.ravel(), minlength=E).astype(np.float64)
    if len(idx) and E > 1:
        r["cv_counts"] = float(counts.std(ddof=1) / counts.mean())
    return r


def _balance_cv_not_squared(p, idx, E):
    r = _orig["balance_losses"](p, idx, E)
    r["cv2_probs"] = float(np.sqrt(r["cv2_probs"]))
    return r


def _balance_first_choices_only(p, idx, E):
    r = _orig["balance_losses"](p, idx, E)
    if len(idx):
        f = np.bincount(idx[:, 0], minlength=E) / len(idx)
        r["aux_all_choices"] = float(E * np.sum(f * p.mean(axis=0)))
    return r


def _shared_only_for_kept_tokens(*args, shared=None, **kw):
    r = _orig["moe_forward"](*args, shared=None, **kw)
    if shared is not None:
        full = _orig["moe_forward"](*args, shared=shared, **kw)
        keep = r["kept"][r["rows"]].any(axis=1)
        r["y"] = np.where(keep[:, None], full["y"], r["y"])
    return r


def _shared_weighted_by_gate(*args, shared=None, **kw):
    r = _orig["moe_forward"](*args, shared=None, **kw)
    if shared is not None:
        full = _orig["moe_forward"](*args, shared=shared, **kw)
        r["y"] = r["y"] + r["gate"][r["rows"], :1] * (full["y"] - r["y"])
    return r


_orig = {n: getattr(M, n) for n in ("top_k", "gates", "expert_ffn", "aux_and_z", "assign_slots", "router_logits",
                                     "balance_losses", "moe_forward")}

MUTANTS = {
    "top_k ties to the higher index": ("top_k", _top_k_last_index_on_ties),
    "renormalised gates left unnormalised": ("gates", _gates_not_renormalised),
    "silu with the wrong sign": ("expert_ffn", _ffn_silu_sign),
    "SwiGLU gate/value roles swapped": ("expert_ffn", _ffn_w1_w3_swapped_roles),
    "aux without the factor E": ("aux_and_z", _aux_without_E),
    "z-loss without the square": ("aux_and_z", _z_without_square),
    "f over all k choices": ("aux_and_z", _f_over_all_choices),
    "capacity off by one": ("assign_slots", _slots_off_by_one),
    "slots by choice before token": ("assign_slots", _slots_choice_major),
    "router weight transposed": ("router_logits", _logits_transposed_router),
    "router bias dropped": ("router_logits", _logits_dropped_bias),
    "CV with the sample standard deviation": ("balance_losses", _balance_sample_std),
    "cv^2 left unsquared": ("balance_losses", _balance_cv_not_squared),
    "all-choices loss over first choices": ("balance_losses", _balance_first_choices_only),
    "shared experts skipped for dropped tokens": ("moe_forward", _shared_only_for_kept_tokens),
    "shared experts scaled by the gate": ("moe_forward", _shared_weighted_by_gate),
}

PINS = [
    lambda O: [P.test_top_k_matches_brute_force_with_ties(O, E) for E in (3, 5)],
    P.test_top_k_signed_zero_is_a_tie,
    P.test_renorm_gates_sum_to_one_and_equal_conditional_probabilities,
    P.test_switch_gate_is_max_probability_below_one,
    P.test_closed_form_golden_routing,
    P.test_router_logits_match_linear_and_are_order_free_on_dyadic_inputs,
    P.test_aux_is_one_under_uniform_routing,
    P.test_aux_tends_to_E_when_collapsed,
    P.test_z_loss_closed_form,
    P.test_dropless_keeps_everything,
    lambda O: P.test_position_order_dropping_k1(O, 3),
    P.test_slot_priority_is_token_order_across_choices,
    P.test_worked_example_reconstruction,
    lambda O: [P.test_single_expert_is_the_dense_ffn(O, a, g) for a in (0, 1) for g in (0, 1)],
    lambda O: [P.test_k_equals_E_is_the_dense_softmax_mixture(O, a) for a in (0, 1)],
    P.test_balance_losses_are_zero_and_one_under_uniform_routing,
    P.test_balance_losses_closed_forms_when_collapsed,
    P.test_all_choices_loss_equals_switch_loss_at_k1_and_counts_every_choice,
    lambda O: [P.test_shared_expert_with_silent_routed_experts_is_the_dense_ffn(O, a) for a in (0, 1)],
    P.test_shared_copy_of_the_single_expert_doubles_the_output,
    P.test_dropped_tokens_still_get_the_shared_experts,
]


def _pins_caught(O):
    caught = 0
    for pin in PINS:
        try:
            pin(O)
        except (AssertionError, ValueError, IndexError):
            caught += 1
    return caught


def test_every_pin_passes_on_the_unaltered_oracles():
    assert _pins_caught(oracle) == 0
    assert _pins_caught(oracle_cpp.load()) == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(M, attr, fn)
    monkeypatch.setattr(oracle, attr, fn)
    assert _pins_caught(oracle) >= 1, f"no pin fails for mutant: {name}"


# (description, text of oracle/moe_oracle.cpp, planted replacement)
CPP_MUTANTS = [
    ("top_k ties to the higher index",
     "if (best < 0 || h[e] > h[best]) best = e;", "if (best < 0 || h[e] >= h[best]) best = e;"),
    ("renormalised gates left unnormalised",
     "for (int64_t j = 0; j < k; ++j) g[j] = std::exp(h[idx[j]] - h[idx[0]]) / sum;",
     "for (int64_t j = 0; j < k; ++j) g[j] = p[idx[j]];"),
    ("silu with the wrong sign",
     "hid[f] = a / (1.0 + std::exp(-a)) * b;", "hid[f] = a / (1.0 + std::exp(a)) * b;"),
    ("SwiGLU gate/value roles swapped",
     "hid[f] = a / (1.0 + std::exp(-a)) * b;", "hid[f] = b / (1.0 + std::exp(-b)) * a;"),
    ("ReLU left out", "hid[f] = a > 0.0 ? a : 0.0;", "hid[f] = a;"),
    ("aux without the factor E", "*aux = E * s;", "*aux = s;"),
    ("z-loss without the square", "zs += lse[t] * lse[t];", "zs += lse[t];"),
    ("log-sum-exp without the max", "*lse = m + std::log(Z);", "*lse = std::log(Z);"),
    ("f over all k choices",
     "for (int64_t t = 0; t < T; ++t) f[idx[t * k]] += 1.0;",
     "for (int64_t a = 0; a < T * k; ++a) f[idx[a]] += 1.0 / k;"),
    ("capacity off by one",
     "kept[a] = (C < 0 || rank[a] < C) ? 1 : 0;", "kept[a] = (C < 0 || rank[a] <= C) ? 1 : 0;"),
    ("offsets from the counts before capacity",
     "offsets[e + 1] = offsets[e] + kept_counts[e];", "offsets[e + 1] = offsets[e] + counts[e];"),
    ("slots by choice before token",
     "  for (int64_t t = 0; t < T; ++t) {\n    for (int64_t j = 0; j < k; ++j) {\n      const int64_t a = t * k + j;",
     "  for (int64_t j = 0; j < k; ++j) {\n    for (int64_t t = 0; t < T; ++t) {\n      const int64_t a = t * k + j;"),
    ("router weight transposed",
     "s += W_r.at(e * d + c) * x.at(t * d + c);", "s += W_r.at(c * E + e) * x.at(t * d + c);"),
    ("router bias dropped", "if (!b_r.null()) s += b_r.at(e);", ""),
    ("CV with the sample standard deviation", "var_c /= E;", "var_c /= (E - 1);"),
    ("cv^2 left unsquared",
     "out[2] = var_p / (mean_p * mean_p);", "out[2] = std::sqrt(var_p) / mean_p;"),
    ("all-choices loss over first choices",
     "for (int64_t a = 0; a < T * k; ++a) c[idx[a]] += 1.0;",
     "for (int64_t t = 0; t < T; ++t) c[idx[t * k]] += k;"),
    ("shared experts skipped for dropped tokens",
     "for (int64_t s = 0; s < n_shared; ++s) {  // shared experts, after the routed sum",
     "bool any_kept = false;\n    for (int64_t j = 0; j < k; ++j) any_kept = any_kept || r->kept[t * k + j];\n"
     "    for (int64_t s = 0; any_kept && s < n_shared; ++s) {"),
    ("shared experts scaled by the gate",
     "      for (int64_t c = 0; c < d; ++c) y[c] += out[c];",
     "      for (int64_t c = 0; c < d; ++c) y[c] += r->gate[t * k] * out[c];"),
]


@pytest.mark.parametrize("case", CPP_MUTANTS, ids=[c[0] for c in CPP_MUTANTS])
def test_cpp_mutant_is_caught(case, tmp_path):
    name, old, new = case
    with open(oracle_cpp.SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutant text not found once in the C++ oracle: {name}"
    path = tmp_path / "mutant.cpp"
    path.write_text(src.replace(old, new))
    lib = oracle_cpp.compile_library(str(path), str(tmp_path / "libmutant.so"), opt="-O1")
    assert _pins_caught(oracle_cpp.load(lib)) >= 1, f"no pin fails for C++ mutant: {name}"
