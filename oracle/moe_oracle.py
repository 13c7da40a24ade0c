"""CPU oracle for the sparse Mixture-of-Experts layer forward pass.

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or run this module; the product
path (the CUDA library and its Python binding) never does.

It is a plain, slow, float64 NumPy restatement of the layer defined on the
page "Mixture of experts" (rayaq.ca/ml-models/mixture-of-experts):

  * section "Replacing the feed-forward block", eq. h = W_r x, p = softmax(h),
    y = sum_{i in TopK(h)} g_i(x) E_i(x);
  * section "Top-k gating": keep the k largest logits, largest first; Switch
    gate (k = 1) = the chosen expert's full-softmax probability; renormalised
    gate = softmax over the k chosen logits;
  * section "The load-balancing loss": L_aux / alpha = E * sum_i f_i P_i with
    f_i the share of tokens whose top choice is i and P_i the mean router
    probability; router z-loss = mean over tokens of (log sum_j exp h_j)^2;
  * section "Capacity and dropped tokens": capacity = tokens/experts x
    capacity factor; slots are filled in position order and the overflow is
    dropped (the layer's output for a dropped assignment is zero; the caller's
    residual carries the input);
  * section "Implementation": SwiGLU expert w2(silu(w1 x) * w3 x); the router
    is computed in float32; the gated expert outputs are summed per token.

Readings where the page is silent (each is listed with its reason in the
design notes of this repository):
  - ties in top-k go to the lower expert index;
  - capacity C = ceil(capacity_factor * T * k / E) (equal to the page's
    formula at k = 1); capacity_factor <= 0 means dropless;
  - slot priority is token order alone (a token's second choice can take a
    slot before a later token's first choice);
  - f_i counts first choices of all T tokens before any dropping; P_i is the
    full softmax over all E experts;
  - gates are not renormalised after drops;
  - the ReLU expert is w2(relu(w1 x)) (the feed-forward block of the same
    page's "Problem" section, with no biases, like the SwiGLU listing);
  - router logits are rounded once to fp32 and every routing decision is
    taken on those fp32 values.

Parity pins: every function here is pinned by tests/test_oracle_pins.py
against closed forms, brute force, library routines and the page's stated
special cases (see that file's docstrings).
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

ACT_RELU, ACT_SWIGLU = 0, 1
GATE_SWITCH, GATE_RENORM = 0, 1


def router_logits(x, W_r, b_r=None, dtype=np.float32) -> np.ndarray:
    """Router logits h = W_r x (+ b) per token, as fp32.

    "Replacing the feed-forward block": the router is one linear layer with E
    rows.  Accumulated in float64 and rounded once to float32 ("compute the
    router in float32", section "Implementation").
    x: [T][d], W_r: [E][d], b_r: [E] or None.  Returns float32 [T][E].
    dtype=np.float64 skips the rounding (for finite-difference checks, whose
    steps are far below float32 resolution).
    """
    h = np.asarray(x, np.float64) @ np.asarray(W_r, np.float64).T
    if b_r is not None:
        h = h + np.asarray(b_r, np.float64)[None, :]
    return h.astype(dtype)


def softmax_lse(h32: np.ndarray):
    """Full softmax p over the E experts and the log-sum-exp of each token.

    p = softmax(h) ("Replacing the feed-forward block"); lse = log sum_j exp h_j
    (the z-loss term of "The load-balancing loss").  float64 from the fp32 logits.
    """
    h = np.asarray(h32, np.float64)
    if h.shape[0] == 0:
        return np.zeros_like(h), np.zeros(0)
    m = h.max(axis=1, keepdims=True)
    e = np.exp(h - m)
    Z = e.sum(axis=1, keepdims=True)
    return e / Z, (m + np.log(Z))[:, 0]


def top_k(h32: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits of each token, largest first.

    "Top-k gating": the router keeps the k largest logits.  Selection is done
    k times on the fp32 values: take the largest remaining logit; among equal
    logits (+0 and -0 compare equal) the lower expert index wins.
    Returns int64 [T][k].
    """
    h = np.asarray(h32, np.float64).copy()
    T = h.shape[0]
    idx = np.empty((T, k), np.int64)
    rows = np.arange(T)
    for j in range(k):
        sel = np.argmax(h, axis=1)  # first index among equal maxima
        idx[:, j] = sel
        h[rows, sel] = -np.inf
    return idx


def gates(h32: np.ndarray, p: np.ndarray, idx: np.ndarray, gate_mode: int) -> np.ndarray:
    """Gate value of each chosen expert ("Top-k gating").

    SWITCH: g_j = p[idx_j], the full-softmax probability (below 1 for E > 1).
    RENORM: g = softmax over the k chosen logits, which equals the chosen
    full-softmax probabilities divided by their sum.
    Returns float64 [T][k].
    """
    rows = np.arange(idx.shape[0])[:, None]
    if gate_mode == GATE_SWITCH:
        return p[rows, idx]
    sel = np.asarray(h32, np.float64)[rows, idx]
    if sel.shape[0] == 0:
        return sel
    e = np.exp(sel - sel[:, :1])  # idx[:, 0] holds the largest logit
    return e / e.sum(axis=1, keepdims=True)


def expert_capacity(capacity_factor: float, T: int, k: int, E: int) -> Optional[int]:
    """Slots per expert ("Capacity and dropped tokens").

    The page's rule is tokens/experts x capacity factor; with k assignments per
    token the assignments per expert are T*k/E, so C = ceil(cf * T * k / E)
    (identical at k = 1).  cf <= 0 means no capacity limit (dropless).
    """
    if capacity_factor <= 0:
        return None
    return int(math.ceil(float(capacity_factor) * T * k / E))


def assign_slots(idx: np.ndarray, E: int, C: Optional[int]):
    """Capacity enforcement with position-order dropping.

    "Capacity and dropped tokens": an expert's slots are filled in position
    order and the assignments beyond its capacity are dropped.  The rank of
    assignment (t, j) is the number of earlier assignments to the same expert
    in token order (a token holds each expert at most once).  Kept iff
    rank < C.  The kept assignments of expert e occupy rows
    offsets[e] .. offsets[e+1]-1 of the expert-sorted dispatch buffer, in token
    order; dest_row is that row, or -1 when dropped.
    """
    T, k = idx.shape
    flat = idx.reshape(-1)
    rank = np.zeros(flat.shape, np.int64)
    counts = np.zeros(E, np.int64)
    for e in range(E):
        hit = flat == e
        n = int(hit.sum())
        rank[hit] = np.arange(n)
        counts[e] = n
    kept = np.ones(flat.shape, bool) if C is None else rank < C
    kept_counts = counts if C is None else np.minimum(counts, C)
    offsets = np.concatenate([[0], np.cumsum(kept_counts)]).astype(np.int64)
    dest = np.where(kept, offsets[flat] + rank, -1)
    return {
        "counts": counts,
        "kept_counts": kept_counts,
        "offsets": offsets,
        "rank": rank.reshape(T, k),
        "kept": kept.reshape(T, k),
        "dest_row": dest.reshape(T, k),
        "dropped": int((~kept).sum()),
    }


def expert_ffn(xr: np.ndarray, W1e, W3e, W2e, act: int) -> np.ndarray:
    """One expert on a batch of rows.

    SWIGLU ("Implementation"): w2(silu(w1 x) * w3 x), silu(u) = u / (1 + e^-u).
    RELU: w2(relu(w1 x)).  Weights in nn.Linear (out, in) layout:
    W1e/W3e [d_ff][d], W2e [d][d_ff].  float64 throughout: the hidden
    activation is never rounded (the page fixes only the router's precision).
    """
    a = xr @ np.asarray(W1e, np.float64).T
    if act == ACT_RELU:
        hdn = np.maximum(a, 0.0)
    else:
        b = xr @ np.asarray(W3e, np.float64).T
        hdn = a / (1.0 + np.exp(-a)) * b
    return hdn @ np.asarray(W2e, np.float64).T


def aux_and_z(p: np.ndarray, lse: np.ndarray, idx: np.ndarray, E: int):
    """Unscaled load-balancing loss and router z-loss ("The load-balancing loss").

    aux = E * sum_i f_i P_i, f_i = share of the T tokens whose first choice is
    i (counted before capacity), P_i = mean full-softmax probability of i.
    z = mean over tokens of lse^2.  The caller applies alpha = 0.01 and 1e-3.
    T = 0 gives aux = z = 0.
    """
    T = p.shape[0]
    if T == 0:
        return 0.0, 0.0
    f = np.bincount(idx[:, 0], minlength=E).astype(np.float64) / T
    P = p.mean(axis=0)
    return float(E * np.sum(f * P)), float(np.mean(lse ** 2))


def balance_losses(p: np.ndarray, idx: np.ndarray, E: int) -> dict:
    """Alternative load-balancing statistics, unscaled (the caller applies its
    coefficient, e.g. 0.01).

    * ``cv_counts``: the coefficient of variation (standard deviation over
      mean, over the E experts) of the expert assignment counts, all k choices
      counted before capacity -- page "Mixture of Experts (MoE)"
      (inferensys.com, self-hosted large language models), training-challenge
      bullets: "a coefficient of 0.01 multiplied by the coefficient of
      variation of expert assignment counts".
    * ``cv2_probs``: the squared coefficient of variation of the router
      probabilities aggregated per expert (P_i, the mean full-softmax
      probability) -- page "Mixture of Experts (MoE) Language Models"
      (chipfoundryservices.com), "Load Balancing and Training": cv^2 of the
      router probabilities.
    * ``aux_all_choices``: the Switch loss of "Mixture of experts" (rayaq.ca),
      section "The load-balancing loss", with f_i the share of all T*k
      assignments (not only first choices) routed to i.

    Readings: standard deviation and variance are of the E values themselves
    (population moments, divided by E); T = 0 gives zeros.
    """
    T, k = idx.shape
    if T == 0:
        return {"aux_all_choices": 0.0, "cv_counts": 0.0, "cv2_probs": 0.0}
    counts = np.bincount(idx.ravel(), minlength=E).astype(np.float64)
    P = p.astype(np.float64).mean(axis=0)
    mean_c = counts.mean()
    cv_counts = float(np.sqrt(np.mean((counts - mean_c) ** 2)) / mean_c)
    mean_p = P.mean()
    cv2_probs = float(np.mean((P - mean_p) ** 2) / mean_p ** 2)
    aux_all = float(E * np.sum(counts / (T * k) * P))
    return {"aux_all_choices": aux_all, "cv_counts": cv_counts, "cv2_probs": cv2_probs}


def moe_forward(x, W_r, b_r, W1, W3, W2, *, k: int, gate_mode: int, act: int,
                capacity_factor: float, rows: Optional[Sequence[int]] = None,
                logits: Optional[np.ndarray] = None,
                shared: Optional[tuple] = None, logits_dtype=np.float32) -> dict:
    """The whole layer: routing for every token, y for every token or for ``rows``.

    x: [T][d]; W_r: [E][d]; b_r: [E] or None; W1, W3: [E][d_ff][d] (W3 None for
    ReLU); W2: [E][d][d_ff]; any float dtype (bf16 values come in widened).
    ``logits``: route from these fp32 logits instead of computing W_r x.
    ``rows``: compute y only for these tokens (routing, capacity and losses are
    always global; y_t depends on x_t and the global routing only).
    ``logits_dtype``: np.float64 keeps the logits unrounded (finite differences).
    ``shared``: (W1s, W3s, W2s), each with n_s experts shaped like W1, W3, W2:
    shared experts that every token visits ("Mixture of experts", section
    "Total versus active parameters": "shared experts every token visits").
    Reading: a shared expert is an FFN of the same shape and activation as the
    routed ones, applied to every token with weight 1, outside routing,
    capacity and the losses; its output is added after the routed sum, in
    shared-expert order, so a token whose routed assignments were all dropped
    still gets it.

    y_t = sum over kept assignments (t, j), in slot order j, of
    g_tj * E_{idx_tj}(x_t), plus sum_s S_s(x_t); a token with all routed
    assignments dropped and no shared experts gets y_t = 0.
    """
    x = np.asarray(x)
    T = x.shape[0]
    E = np.asarray(W_r).shape[0]
    h32 = router_logits(x, W_r, b_r, logits_dtype) if logits is None else np.asarray(logits, logits_dtype)
    p, lse = softmax_lse(h32)
    idx = top_k(h32, k)
    g = gates(h32, p, idx, gate_mode)
    C = expert_capacity(capacity_factor, T, k, E)
    slots = assign_slots(idx, E, C)
    aux, z = aux_and_z(p, lse, idx, E)

    want = np.arange(T) if rows is None else np.asarray(rows, np.int64)
    d = x.shape[1]
    # contrib[i, j] = g_tj * E_{idx_tj}(x_t) for token t = want[i] (0 if dropped)
    contrib = np.zeros((len(want), k, d), np.float64)
    ew = idx[want]                      # [n][k] experts of the wanted tokens
    kw = slots["kept"][want]            # [n][k] kept flags
    for e in range(E):
        ii, jj = np.nonzero((ew == e) & kw)
        if ii.size == 0:
            continue
        ts = want[ii]
        out = expert_ffn(np.asarray(x[ts], np.float64), W1[e],
                         None if W3 is None else W3[e], W2[e], act)
        contrib[ii, jj] = g[ts, jj][:, None] * out
    y = np.zeros((len(want), d), np.float64)
    for j in range(k):                  # slot order
        y += contrib[:, j]
    if shared is not None:
        W1s, W3s, W2s = shared
        xs = np.asarray(x[want], np.float64)
        for si in range(len(W1s)):      # shared-expert order, after the routed sum
            y += expert_ffn(xs, W1s[si], None if W3s is None else W3s[si], W2s[si], act)
    res = {"logits": h32, "p": p, "lse": lse, "idx": idx, "gate": g, "capacity": C,
           "y": y, "rows": want, "aux": aux, "z": z}
    res.update(balance_losses(p, idx, E))
    res.update(slots)
    return res


# ----------------------------------------------------------------------------- 4-bit weights
# "Mixture of Experts (MoE)" (inferensys.com, inference-optimization glossary),
# model quantization paragraph: post-training quantization of a trained MoE's
# weights to 4-bit integers; "Mixture of experts" (rayaq.ca), "Total versus
# active parameters": small-batch decoding is bound by reading expert weights,
# which quantization eases.  The pages fix no scheme; the reading here:
#   * symmetric per-group quantization along the input dimension K of each
#     weight row, groups of INT4_GROUP consecutive elements;
#   * scale s = max|w| / 7 over the group, computed in float32 and rounded UP
#     to 5 significant bits (so that every code times s is exact in bfloat16);
#   * code q = round-half-even(w / s) in float32 (|w / s| <= 7, so q in [-7, 7];
#     the stored range is [-8, 7]); s = 0 (an all-zero group) gives q = 0;
#   * the dequantized weight is q * s, exactly.
# Storage: codes u = q + 8 in 4 bits; each 32-bit word holds 8 consecutive
# elements k0..k7 of a row, element k_{2j} in bits 4j..4j+3 and element
# k_{2j+1} in bits 4j+16..4j+19 (j = 0..3); words stored in tiles of 128 rows x
# 64 elements, [rows / 128][K / 64][128 rows][8 words]; scales are bfloat16,
# [rows / 128][K / INT4_GROUP][128 rows].
INT4_GROUP = 128


def _round_up_5_significant_bits(s32: np.ndarray) -> np.ndarray:
    """Smallest float32 with at most 5 significant bits that is >= s (s >= 0)."""
    u = np.asarray(s32, np.float32).view(np.uint32).astype(np.uint64)
    low = u & ((1 << 19) - 1)
    u = np.where(low != 0, (u | ((1 << 19) - 1)) + 1, u)
    return u.astype(np.uint32).view(np.float32)


def quantize_int4(W) -> tuple:
    """Codes q [rows][K] (int8, -8..7) and float32 scales [rows][K / INT4_GROUP]
    of a weight matrix W [rows][K] (bfloat16 values given as floats), by the
    rule above; K must be a multiple of INT4_GROUP."""
    W = np.asarray(W, np.float32)
    rows, K = W.shape
    assert K % INT4_GROUP == 0
    g = W.reshape(rows, K // INT4_GROUP, INT4_GROUP)
    amax = np.abs(g).max(axis=2).astype(np.float32)
    s = _round_up_5_significant_bits((amax / np.float32(7.0)).astype(np.float32))
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(s[:, :, None] > 0, np.rint((g / s[:, :, None]).astype(np.float32)), 0.0)
    q = np.clip(r, -8, 7).astype(np.int8).reshape(rows, K)
    return q, s


def pack_int4(q: np.ndarray) -> np.ndarray:
    """Words (uint32, flat, in tiles) of codes q [rows][K] in the storage layout
    above; rows and K multiples of 128."""
    q = np.asarray(q, np.int64)
    rows, K = q.shape
    u = (q + 8).reshape(rows, K // 8, 8).astype(np.uint64)
    w = np.zeros((rows, K // 8), np.uint64)
    for j in range(4):
        w |= u[:, :, 2 * j] << (4 * j)
        w |= u[:, :, 2 * j + 1] << (4 * j + 16)
    # [rows][K/8] -> [rows/128][128][K/64][8] -> [rows/128][K/64][128][8]
    tiles = w.reshape(rows // 128, 128, K // 64, 8).transpose(0, 2, 1, 3)
    return np.ascontiguousarray(tiles).astype(np.uint32).reshape(-1)


def tile_scales(s: np.ndarray) -> np.ndarray:
    """Scales [rows][K / INT4_GROUP] in the storage layout (flat, in tiles)."""
    s = np.asarray(s)
    rows, G = s.shape
    return np.ascontiguousarray(s.reshape(rows // 128, 128, G).transpose(0, 2, 1)).reshape(-1)


def dequantize_int4(words, scales, rows: int, K: int) -> np.ndarray:
    """Weights [rows][K] (float64) from the stored words and scales (flat, in
    tiles): element k of a row = (u_k - 8) * s_{k // INT4_GROUP}."""
    w = np.asarray(words, np.uint64).reshape(rows // 128, K // 64, 128, 8).transpose(0, 2, 1, 3)
    w = w.reshape(rows, K // 8)
    u = np.empty((rows, K // 8, 8), np.int64)
    for j in range(4):
        u[:, :, 2 * j] = (w >> (4 * j)) & 0xF
        u[:, :, 2 * j + 1] = (w >> (4 * j + 16)) & 0xF
    q = (u - 8).reshape(rows, K).astype(np.float64)
    sc = np.asarray(scales, np.float64).reshape(rows // 128, K // INT4_GROUP, 128).transpose(0, 2, 1)
    s = np.repeat(sc.reshape(rows, K // INT4_GROUP), INT4_GROUP, axis=1)
    return q * s
