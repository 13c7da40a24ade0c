"""Pins of the CPU oracle against what the pages and the mathematics fix.

No test here compares the oracle with itself: each check uses a closed form,
brute force, a library routine (torch / scipy) or a value derived by hand from
the page "Mixture of experts" (rayaq.ca), stored under tests/golden/.

Every pin runs against both oracles: the NumPy restatement
(oracle/moe_oracle.py) and the plain C++ loops (oracle/moe_oracle.cpp,
through oracle/cpp.py).
"""
import itertools
import math

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle
from oracle import cpp as oracle_cpp
from tests._golden import load

IMPLS = {"numpy": lambda: oracle, "cpp": lambda: oracle_cpp.load()}


@pytest.fixture(params=sorted(IMPLS))
def O(request):
    """The oracle under test: the NumPy module or the C++ library binding."""
    return IMPLS[request.param]()

rng = np.random.default_rng(7)


# ---------------------------------------------------------------- top-k
@pytest.mark.parametrize("E", [1, 2, 3, 5, 7, 8])
def test_top_k_matches_brute_force_with_ties(O, E):
    """Top-k gating: k largest logits, largest first; ties -> lower index.

    Brute force over all k-subsets: the chosen set has the maximal logit sum,
    and among maximal sets it is the lexicographically smallest; its order is
    (value descending, index ascending).  Logits are drawn from a 5-value set
    (plus -0.0) so ties are frequent.
    """
    vals = np.array([-1.0, -0.5, 0.0, -0.0, 0.5, 1.0], np.float32)
    h = vals[rng.integers(0, len(vals), size=(200, E))]
    for k in range(1, E + 1):
        idx = O.top_k(h, k)
        for t in range(h.shape[0]):
            best = max(itertools.combinations(range(E), k),
                       key=lambda s: (sum(float(h[t, i]) for i in s), [-i for i in s]))
            assert sorted(idx[t].tolist()) == list(best)
            order = sorted(best, key=lambda i: (-float(h[t, i]), i))
            assert idx[t].tolist() == order


def test_top_k_signed_zero_is_a_tie(O):
    h = np.array([[-0.0, 0.0], [0.0, -0.0]], np.float32)
    assert O.top_k(h, 1)[:, 0].tolist() == [0, 0]


# ---------------------------------------------------------------- softmax, lse, logits
def test_softmax_and_lse_match_scipy(O):
    h = rng.normal(size=(50, 9)).astype(np.float32) * 5
    p, lse = O.softmax_lse(h)
    np.testing.assert_allclose(p, scipy.special.softmax(h.astype(np.float64), axis=1), rtol=1e-13)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(h.astype(np.float64), axis=1), rtol=1e-13)


def test_router_logits_match_linear_and_are_order_free_on_dyadic_inputs(O):
    """h = W_r x + b (one linear layer with E rows); dyadic inputs give exact fp32."""
    x = np.clip(np.round(rng.normal(size=(33, 64)) * 64) / 64, -4, 4)
    W = np.clip(np.round(rng.normal(size=(6, 64)) / 8 * 1024) / 1024, -1, 1)
    b = np.round(rng.normal(size=6) * 1024) / 1024
    h = O.router_logits(x, W, b)
    ref = F.linear(torch.tensor(x), torch.tensor(W), torch.tensor(b)).numpy()
    assert np.array_equal(h, ref.astype(np.float32))
    # square, non-symmetric router (d == E): catches a transposed W_r
    Wsq = W[:, :6]
    hs = O.router_logits(x[:, :6], Wsq, None)
    assert np.array_equal(hs, F.linear(torch.tensor(x[:, :6]), torch.tensor(Wsq)).numpy().astype(np.float32))
    # any fp32 summation order gives the same logits
    for _ in range(3):
        perm = rng.permutation(64)
        acc = np.zeros((33, 6), np.float32)
        for c in perm:
            acc = (acc + (x[:, c:c + 1] * W[:, c][None, :]).astype(np.float32)).astype(np.float32)
        assert np.array_equal((acc + b.astype(np.float32)).astype(np.float32), h)


# ---------------------------------------------------------------- gates
def test_renorm_gates_sum_to_one_and_equal_conditional_probabilities(O):
    """Top-k gating, renormalised bullet: g = p_sel / sum(p_sel), sums to 1."""
    h = (rng.normal(size=(40, 8)) * 3).astype(np.float32)
    p = scipy.special.softmax(h.astype(np.float64), axis=1)
    for k in (1, 2, 3, 8):
        idx = O.top_k(h, k)
        g = O.gates(h, p, idx, O.GATE_RENORM)
        np.testing.assert_allclose(g.sum(axis=1), 1.0, rtol=1e-14)
        psel = np.take_along_axis(p, idx, axis=1)
        np.testing.assert_allclose(g, psel / psel.sum(axis=1, keepdims=True), rtol=1e-12)
        assert np.all(np.diff(g, axis=1) <= 1e-15)  # largest first


def test_switch_gate_is_max_probability_below_one(O):
    """Top-k gating, Switch bullet: gate = the argmax expert's full-softmax p < 1."""
    h = (rng.normal(size=(40, 8)) * 3).astype(np.float32)
    p = scipy.special.softmax(h.astype(np.float64), axis=1)
    idx = O.top_k(h, 1)
    g = O.gates(h, p, idx, O.GATE_SWITCH)
    np.testing.assert_allclose(g[:, 0], p.max(axis=1), rtol=1e-15)
    assert np.all(g < 1.0)


def test_closed_form_golden_routing(O):
    G = load("closed_form_routing.txt")
    h = np.array([G["logits_t0"], G["logits_t1"]], np.float32)
    p, lse = O.softmax_lse(h)
    np.testing.assert_allclose(p, [G["p_t0"], G["p_t1"]], rtol=1e-6)
    np.testing.assert_allclose(lse, G["lse"], rtol=1e-6)
    idx2 = O.top_k(h, 2)
    assert idx2.tolist() == G["top2_idx"]
    np.testing.assert_allclose(O.gates(h, p, idx2, O.GATE_RENORM), G["top2_renorm_gates"], rtol=1e-6)
    idx1 = O.top_k(h, 1)
    assert idx1.tolist() == G["top1_idx"]
    np.testing.assert_allclose(O.gates(h, p, idx1, O.GATE_SWITCH), G["top1_switch_gates"], rtol=1e-6)
    aux, z = O.aux_and_z(p, lse, idx2, 3)
    assert aux == pytest.approx(G["aux"], rel=1e-6)
    assert z == pytest.approx(G["z"], rel=1e-6)
    # the same through the whole layer, routing from the given logits
    x = np.zeros((2, 4))
    W1 = np.zeros((3, 5, 4)); W2 = np.zeros((3, 4, 5))
    r = O.moe_forward(x, np.zeros((3, 4)), None, W1, None, W2, k=2, gate_mode=O.GATE_RENORM,
                      act=O.ACT_RELU, capacity_factor=0.0, logits=h)
    assert r["aux"] == pytest.approx(G["aux"], rel=1e-6)
    assert r["z"] == pytest.approx(G["z"], rel=1e-6)


# ---------------------------------------------------------------- losses
def test_aux_is_one_under_uniform_routing(O):
    """The load-balancing loss: uniform first choices give E*sum f P = 1 (so alpha*1)."""
    for E in (2, 4, 8, 64):
        T = 4 * E
        x = np.zeros((T, E)); x[np.arange(T), np.arange(T) % E] = 3.0
        r = O.moe_forward(x, np.eye(E), None, np.zeros((E, 2, E)), None, np.zeros((E, E, 2)),
                          k=1, gate_mode=O.GATE_SWITCH, act=O.ACT_RELU, capacity_factor=0.0)
        assert r["aux"] == pytest.approx(1.0, abs=1e-12)
        assert 0.01 * r["aux"] == pytest.approx(0.01, abs=1e-14)


def test_aux_tends_to_E_when_collapsed(O):
    """Every token to one expert with probability ~1 gives E*sum f P -> E."""
    E, T = 8, 32
    x = rng.normal(size=(T, 16))
    W = rng.normal(size=(E, 16)) * 1e-3
    b = np.zeros(E); b[3] = 40.0
    r = O.moe_forward(x, W, b, np.zeros((E, 2, 16)), None, np.zeros((E, 16, 2)),
                      k=2, gate_mode=O.GATE_RENORM, act=O.ACT_RELU, capacity_factor=0.0)
    assert np.all(r["idx"][:, 0] == 3)
    assert r["aux"] == pytest.approx(E, rel=1e-12)


def test_z_loss_closed_form(O):
    """All logits equal to c: lse = c + ln E, so z = (c + ln E)^2."""
    for E, c in [(4, 0.0), (8, 2.5), (128, -3.0)]:
        h = np.full((5, E), c, np.float32)
        p, lse = O.softmax_lse(h)
        _, z = O.aux_and_z(p, lse, O.top_k(h, 1), E)
        assert z == pytest.approx((c + math.log(E)) ** 2, rel=1e-12)


def test_balance_losses_are_zero_and_one_under_uniform_routing(O):
    """Uniform routing: equal assignment counts and equal P_i give a coefficient
    of variation 0, cv^2 0, and the all-choices Switch loss E*sum f P = 1."""
    for E, k in [(4, 1), (8, 2), (16, 4)]:
        T = 8 * E
        idx = np.stack([(np.arange(T) + j) % E for j in range(k)], axis=1)  # each expert k*T/E times
        p = np.full((T, E), 1.0 / E)
        r = O.balance_losses(p, idx, E)
        assert r["cv_counts"] == pytest.approx(0.0, abs=1e-15)
        assert r["cv2_probs"] == pytest.approx(0.0, abs=1e-15)
        assert r["aux_all_choices"] == pytest.approx(1.0, abs=1e-12)


def test_balance_losses_closed_forms_when_collapsed(O):
    """All T tokens to expert 0 with probability 1 (k = 1): counts (T, 0, ..., 0)
    have mean T/E and standard deviation (T/E) sqrt(E - 1), so CV = sqrt(E - 1);
    P = e_0 gives cv^2 = E - 1; the all-choices loss equals E."""
    for E in (2, 5, 8, 64):
        T = 3 * E
        idx = np.zeros((T, 1), np.int64)
        p = np.zeros((T, E)); p[:, 0] = 1.0
        r = O.balance_losses(p, idx, E)
        assert r["cv_counts"] == pytest.approx(math.sqrt(E - 1), rel=1e-12)
        assert r["cv2_probs"] == pytest.approx(E - 1, rel=1e-12)
        assert r["aux_all_choices"] == pytest.approx(E, rel=1e-12)


def test_all_choices_loss_equals_switch_loss_at_k1_and_counts_every_choice(O):
    """k = 1: first choices are all choices, so the two losses agree; k = 2 with
    second choices on one expert: f over all choices differs from first choices."""
    E, T, d = 6, 40, 9
    x = rng.normal(size=(T, d)); W_r = rng.normal(size=(E, d))
    z = np.zeros((E, 2, d)), np.zeros((E, d, 2))
    r = O.moe_forward(x, W_r, None, z[0], None, z[1], k=1, gate_mode=O.GATE_SWITCH, act=O.ACT_RELU,
                      capacity_factor=0.0)
    assert r["aux_all_choices"] == pytest.approx(r["aux"], rel=1e-12)
    # hand-made: first choices uniform over experts 0..3, every second choice = expert 5
    T2 = 8
    idx = np.stack([np.arange(T2) % 4, np.full(T2, 5)], axis=1)
    P = np.arange(1.0, E + 1) / np.sum(np.arange(1.0, E + 1))   # non-uniform, so f matters
    p = np.tile(P, (T2, 1))
    bl = O.balance_losses(p, idx, E)
    counts = np.array([2, 2, 2, 2, 0, 8], float)
    assert bl["aux_all_choices"] == pytest.approx(E * np.sum(counts / 16 * P), rel=1e-12)
    assert bl["aux_all_choices"] != pytest.approx(E * np.sum(np.array([2, 2, 2, 2, 0, 0]) / 8 * P), rel=1e-6)
    assert bl["cv_counts"] == pytest.approx(counts.std() / counts.mean(), rel=1e-12)


# ---------------------------------------------------------------- capacity
def test_capacity_formula(O):
    """Capacity and dropped tokens: C = tokens/experts x factor (x k for top-k)."""
    assert O.expert_capacity(1.25, 8192, 1, 64) == 160
    assert O.expert_capacity(2.0, 16384, 4, 128) == 1024
    assert O.expert_capacity(1.0, 8, 1, 4) == 2
    assert O.expert_capacity(1.0, 10, 1, 4) == 3  # ceil
    assert O.expert_capacity(0.0, 10, 2, 4) is None
    assert O.expert_capacity(-1.0, 10, 2, 4) is None


def test_dropless_keeps_everything(O):
    idx = rng.integers(0, 5, size=(300, 1))
    s = O.assign_slots(idx, 5, None)
    assert s["dropped"] == 0 and s["kept"].all()
    assert s["kept_counts"].tolist() == np.bincount(idx[:, 0], minlength=5).tolist()


@pytest.mark.parametrize("C", [1, 3, 17])
def test_position_order_dropping_k1(O, C):
    """Slots fill in position order: the kept tokens of an expert are its first C."""
    T, E = 400, 6
    idx = rng.integers(0, E, size=(T, 1))
    s = O.assign_slots(idx, E, C)
    for e in range(E):
        toks = np.sort(np.nonzero(idx[:, 0] == e)[0])
        kept = np.nonzero(s["kept"][:, 0] & (idx[:, 0] == e))[0]
        assert kept.tolist() == toks[:C].tolist()
        rows = s["dest_row"][kept, 0]
        assert rows.tolist() == list(range(s["offsets"][e], s["offsets"][e] + len(kept)))
    assert s["kept"].sum() + s["dropped"] == T


def test_slot_priority_is_token_order_across_choices(O):
    """A token's second choice takes a slot before a later token's first choice."""
    idx = np.array([[1, 0], [0, 2], [0, 1]])  # expert 0: (t0,j1), (t1,j0), (t2,j0)
    s = O.assign_slots(idx, 3, 2)
    assert s["kept"].tolist() == [[True, True], [True, True], [False, True]]
    assert s["dropped"] == 1
    assert s["counts"].tolist() == [3, 2, 1]
    assert s["offsets"].tolist() == [0, 2, 4, 5]
    assert s["dest_row"].tolist() == [[2, 0], [1, 4], [-1, 3]]


def test_worked_example_reconstruction(O):
    G = load("worked_example_capacity.txt")
    idx = np.array(G["first_choice"])[:, None]
    for cf, cap, drops in [(1.0, G["cf1_capacity"], G["cf1_dropped_tokens"]),
                           (2.0, G["cf2_capacity"], G["cf2_dropped_tokens"])]:
        C = O.expert_capacity(cf, G["T"], G["k"], G["E"])
        assert C == cap
        s = O.assign_slots(idx, G["E"], C)
        assert np.nonzero(~s["kept"][:, 0])[0].tolist() == drops
    s2 = O.assign_slots(idx, G["E"], G["cf2_capacity"])
    empty = [1 - s2["kept_counts"][e] / G["cf2_capacity"] for e in (1, 2, 3)]
    assert empty == G["cf2_empty_fraction_experts_1_to_3"]
    s1 = O.assign_slots(idx, G["E"], G["cf1_capacity"])
    assert s1["dropped"] - s2["dropped"] == 2  # "saves two of them"


# ---------------------------------------------------------------- whole-layer reductions
def _torch_ffn(x, W1, W3, W2, act):
    a = F.linear(x, W1)
    hdn = F.relu(a) if act == oracle.ACT_RELU else F.silu(a) * F.linear(x, W3)
    return F.linear(hdn, W2)


@pytest.mark.parametrize("act", [oracle.ACT_RELU, oracle.ACT_SWIGLU])
@pytest.mark.parametrize("gate_mode", [oracle.GATE_RENORM, oracle.GATE_SWITCH])
def test_single_expert_is_the_dense_ffn(O, act, gate_mode):
    """E = 1, k = 1: the router always picks the only expert with gate 1 -> dense FFN."""
    T, d, dff = 23, 12, 20
    x = rng.normal(size=(T, d)); W_r = rng.normal(size=(1, d))
    W1 = rng.normal(size=(1, dff, d)); W3 = rng.normal(size=(1, dff, d)); W2 = rng.normal(size=(1, d, dff))
    r = O.moe_forward(x, W_r, None, W1, W3 if act else None, W2, k=1, gate_mode=gate_mode,
                      act=act, capacity_factor=0.0)
    ref = _torch_ffn(torch.tensor(x), torch.tensor(W1[0]), torch.tensor(W3[0]), torch.tensor(W2[0]), act)
    np.testing.assert_allclose(r["y"], ref.numpy(), rtol=1e-12, atol=1e-12)
    assert r["gate"].tolist() == [[1.0]] * T


@pytest.mark.parametrize("act", [oracle.ACT_RELU, oracle.ACT_SWIGLU])
def test_k_equals_E_is_the_dense_softmax_mixture(O, act):
    """k = E, no capacity: y = sum_e softmax(h)_e E_e(x), every expert weighted."""
    T, d, dff, E = 17, 10, 14, 5
    x = rng.normal(size=(T, d)); W_r = rng.normal(size=(E, d)); b = rng.normal(size=E)
    W1 = rng.normal(size=(E, dff, d)); W3 = rng.normal(size=(E, dff, d)); W2 = rng.normal(size=(E, d, dff))
    r = O.moe_forward(x, W_r, b, W1, W3 if act else None, W2, k=E, gate_mode=O.GATE_RENORM,
                      act=act, capacity_factor=0.0)
    h = F.linear(torch.tensor(x), torch.tensor(W_r), torch.tensor(b)).float().double()
    p = torch.softmax(h, dim=-1)
    ref = sum(p[:, e:e + 1] * _torch_ffn(torch.tensor(x), torch.tensor(W1[e]), torch.tensor(W3[e]),
                                         torch.tensor(W2[e]), act) for e in range(E))
    np.testing.assert_allclose(r["y"], ref.numpy(), rtol=1e-10, atol=1e-12)


def test_sampled_rows_equal_full_rows_and_dropped_tokens_are_zero(O):
    T, d, dff, E, k = 60, 8, 12, 4, 2
    x = rng.normal(size=(T, d)); W_r = rng.normal(size=(E, d))
    W1 = rng.normal(size=(E, dff, d)); W2 = rng.normal(size=(E, d, dff))
    full = O.moe_forward(x, W_r, None, W1, None, W2, k=k, gate_mode=O.GATE_RENORM,
                         act=O.ACT_RELU, capacity_factor=0.5)
    assert full["dropped"] > 0
    rows = [0, 5, 59, 31]
    part = O.moe_forward(x, W_r, None, W1, None, W2, k=k, gate_mode=O.GATE_RENORM,
                         act=O.ACT_RELU, capacity_factor=0.5, rows=rows)
    # equal up to fp64 rounding: BLAS may sum a 4-row batch in another order than a 60-row one
    np.testing.assert_allclose(part["y"], full["y"][rows], rtol=1e-13, atol=1e-13)
    gone = ~full["kept"].any(axis=1)
    assert gone.any() and np.all(full["y"][gone] == 0)
    # a partially dropped token keeps its surviving gate as it is (no renormalisation)
    part_drop = np.nonzero(full["kept"].any(axis=1) & ~full["kept"].all(axis=1))[0]
    assert part_drop.size
    t = part_drop[0]; j = int(np.nonzero(full["kept"][t])[0][0]); e = full["idx"][t, j]
    ref = full["gate"][t, j] * O.expert_ffn(x[t:t + 1], W1[e], None, W2[e], O.ACT_RELU)[0]
    np.testing.assert_allclose(full["y"][t], ref, rtol=1e-13)


# ---------------------------------------------------------------- shared experts
@pytest.mark.parametrize("act", [oracle.ACT_RELU, oracle.ACT_SWIGLU])
def test_shared_expert_with_silent_routed_experts_is_the_dense_ffn(O, act):
    """Routed experts whose output is zero (W2 = 0): y is the sum of the shared
    experts' dense FFNs, for every token."""
    T, d, dff, E, ns = 19, 8, 12, 4, 2
    x = rng.normal(size=(T, d)); W_r = rng.normal(size=(E, d))
    W1 = rng.normal(size=(E, dff, d)); W3 = rng.normal(size=(E, dff, d)); W2 = np.zeros((E, d, dff))
    S1 = rng.normal(size=(ns, dff, d)); S3 = rng.normal(size=(ns, dff, d)); S2 = rng.normal(size=(ns, d, dff))
    r = O.moe_forward(x, W_r, None, W1, W3 if act else None, W2, k=2, gate_mode=O.GATE_RENORM, act=act,
                      capacity_factor=0.0, shared=(S1, S3 if act else None, S2))
    ref = sum(_torch_ffn(torch.tensor(x), torch.tensor(S1[s]), torch.tensor(S3[s]), torch.tensor(S2[s]), act)
              for s in range(ns))
    np.testing.assert_allclose(r["y"], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_shared_copy_of_the_single_expert_doubles_the_output(O):
    """E = 1, k = 1 (gate 1) and one shared expert with the same weights: y = 2 FFN(x)."""
    T, d, dff = 11, 6, 10
    x = rng.normal(size=(T, d)); W_r = rng.normal(size=(1, d))
    W1 = rng.normal(size=(1, dff, d)); W2 = rng.normal(size=(1, d, dff))
    r = O.moe_forward(x, W_r, None, W1, None, W2, k=1, gate_mode=O.GATE_RENORM, act=O.ACT_RELU,
                      capacity_factor=0.0, shared=(W1.copy(), None, W2.copy()))
    ref = _torch_ffn(torch.tensor(x), torch.tensor(W1[0]), None, torch.tensor(W2[0]), O.ACT_RELU)
    np.testing.assert_allclose(r["y"], 2 * ref.numpy(), rtol=1e-12, atol=1e-12)


def test_dropped_tokens_still_get_the_shared_experts(O):
    """Capacity drops routed assignments only: a token with every routed choice
    dropped gets exactly the shared output; routing, counts and losses do not
    see the shared experts."""
    T, d, dff, E, k = 50, 8, 12, 4, 2
    x = rng.normal(size=(T, d)); W_r = rng.normal(size=(E, d))
    W1 = rng.normal(size=(E, dff, d)); W2 = rng.normal(size=(E, d, dff))
    S1 = rng.normal(size=(1, dff, d)); S2 = rng.normal(size=(1, d, dff))
    plain = O.moe_forward(x, W_r, None, W1, None, W2, k=k, gate_mode=O.GATE_RENORM, act=O.ACT_RELU,
                          capacity_factor=0.25)
    sh = O.moe_forward(x, W_r, None, W1, None, W2, k=k, gate_mode=O.GATE_RENORM, act=O.ACT_RELU,
                       capacity_factor=0.25, shared=(S1, None, S2))
    gone = ~plain["kept"].any(axis=1)
    assert gone.sum() > 0
    shared_out = _torch_ffn(torch.tensor(x), torch.tensor(S1[0]), None, torch.tensor(S2[0]), O.ACT_RELU).numpy()
    np.testing.assert_allclose(sh["y"][gone], shared_out[gone], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sh["y"], plain["y"] + shared_out, rtol=1e-12, atol=1e-12)
    for key in ("idx", "counts", "dest_row", "kept"):
        np.testing.assert_array_equal(sh[key], plain[key])
    assert (sh["aux"], sh["z"], sh["dropped"]) == (plain["aux"], plain["z"], plain["dropped"])
