"""Pins for the float64 oracle (CPU only).

Each test ties an oracle function to something other than itself: a value the
pages print (fixtures under tests/golden/, each with its citation), a closed
form, an invariant, or brute force on tiny inputs.  They are chosen so that a
plausible slip in the oracle (a dropped term, a wrong sign or index, a
transposed operand, a wrong tie rule) fails one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LN3 = math.log(3.0)


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- gate logits
def test_gate_logits_one_hot_weights_pick_and_scale_inputs():
    # Wg[e, j] = c_e * [j == pi(e)]  =>  logits[t, e] = c_e * x[t, pi(e)] + o_e.
    # Integer-valued inputs keep every product exact.  d != E and pi is not the
    # identity, so a transposed Wg or swapped loop indices give other numbers.
    T, d, E = 5, 7, 3
    rng = np.random.default_rng(0)
    x = rng.integers(-9, 10, size=(T, d)).astype(np.float64)
    pi = [4, 0, 6]
    c = [2.0, -3.0, 0.5]
    wg = np.zeros((E, d))
    for e in range(E):
        wg[e, pi[e]] = c[e]
    off = np.array([0.25, -1.0, 8.0], np.float32)
    got = oracle.gate_logits(x, wg, off)
    for t in range(T):
        for e in range(E):
            assert got[t, e] == c[e] * x[t, pi[e]] + float(off[e])


def test_gate_logits_bf16_and_f32_inputs_are_upcast_exactly():
    import torch
    vals = torch.tensor([[1.0, -2.5, 0.1171875, 3.0]], dtype=torch.bfloat16)
    w = torch.tensor([[1.0, 1.0, 1.0, 1.0]], dtype=torch.bfloat16)
    got = oracle.gate_logits(vals, w)
    assert got[0, 0] == 1.0 - 2.5 + 0.1171875 + 3.0
    got32 = oracle.gate_logits(np.array([[0.1]], np.float32), np.array([[1.0]], np.float32))
    assert got32[0, 0] == float(np.float32(0.1))


# --------------------------------------------------------------------- softmax
def test_softmax_two_experts_is_logistic():
    l = np.array([[0.0, LN3], [2.0, 2.0], [-1.0, 3.0]])
    p = oracle.softmax(l)
    assert p[0, 0] == pytest.approx(0.25, abs=1e-15)
    assert p[0, 1] == pytest.approx(0.75, abs=1e-15)
    assert p[1, 0] == 0.5 and p[1, 1] == 0.5
    assert p[2, 1] == pytest.approx(1.0 / (1.0 + math.exp(-4.0)), rel=1e-15)


def test_softmax_rows_sum_to_one_and_shift_invariant():
    rng = np.random.default_rng(1)
    l = rng.normal(size=(20, 13)) * 5
    p = oracle.softmax(l)
    assert np.allclose(p.sum(1), 1.0, atol=1e-14)
    assert np.allclose(oracle.softmax(l + 123.0), p, atol=1e-14)
    assert (p > 0).all()


def test_softmax_uniform_logits_give_exact_one_over_e():
    for E in (1, 2, 8, 64, 128):
        p = oracle.softmax(np.full((3, E), 0.7))
        assert (p == 1.0 / E).all()


# ------------------------------------------------------------------- selection
def _brute_topk(score, K):
    order = sorted(range(len(score)), key=lambda e: (-score[e], e))
    return order[:K]


@pytest.mark.parametrize("E,K", [(1, 1), (2, 1), (4, 2), (5, 3), (8, 2), (16, 4), (16, 16)])
def test_select_matches_brute_force_sort_on_tiny_inputs(E, K):
    rng = np.random.default_rng(E * 31 + K)
    # small integers: plenty of exact ties, so the tie rule is exercised
    l = rng.integers(-3, 4, size=(200, E)).astype(np.float64)
    idx, w, p = oracle.select(l, K)
    for t in range(l.shape[0]):
        want = _brute_topk(list(l[t]), K)
        assert list(idx[t]) == want
        sel = [math.exp(l[t, e]) for e in want]
        for k in range(K):
            assert w[t, k] == pytest.approx(sel[k] / sum(sel), rel=1e-13)


def test_select_all_equal_logits_take_lowest_indices_with_equal_weights():
    for E, K in [(8, 2), (128, 8), (64, 4)]:
        idx, w, _ = oracle.select(np.zeros((4, E)), K)
        assert (idx == np.arange(K)).all()
        assert np.allclose(w, 1.0 / K, rtol=0, atol=1e-16)


def test_select_golden_mixtral_two_of_eight():
    g = golden("mixtral_gating.json")
    vals = {"0": 0.0, "ln3": LN3, "-1": -1.0, "-2": -2.0, "-3": -3.0, "-5": -5.0}
    l = np.array([[vals[v] for v in g["logits"]]])
    idx, w, _ = oracle.select(l, g["top_k"])
    assert list(idx[0]) == g["expected_idx"]
    want = [float(Fraction(s)) for s in g["expected_w"]]
    assert w[0] == pytest.approx(want, abs=1e-15)


def test_select_weights_renormalise_to_one():
    rng = np.random.default_rng(2)
    l = rng.normal(size=(300, 64)) * 3
    _, w, _ = oracle.select(l, 6)
    assert np.allclose(w.sum(1), 1.0, atol=1e-14)
    assert (np.diff(w, axis=1) <= 1e-16).all()  # listed best-first


def test_select_prob_space_bias_steers_selection_not_weights():
    # p = softmax([0, ln3, 0, 0]) = [1/6, 1/2, 1/6, 1/6].  With b = [0, 0, 0, 0.4]
    # the scores are [1/6, 1/2, 1/6, 17/30]: expert 3 then 1.  Gate weights use
    # the unbiased p: 1/6 and 1/2 renormalised -> 1/4, 3/4.
    l = np.array([[0.0, LN3, 0.0, 0.0]])
    b = np.array([0.0, 0.0, 0.0, 0.4], np.float32)
    idx, w, p = oracle.select(l, 2, bias=b, bias_mode=oracle.BIAS_PROB)
    assert list(idx[0]) == [3, 1]
    assert w[0] == pytest.approx([0.25, 0.75], abs=1e-15)
    # bias 0.2 on expert 3 in probability space is not enough (1/6+0.2 < 1/2)
    # but in logit space it beats expert 0's logit and loses to ln 3.
    b2 = np.array([0.0, 0.0, 0.0, 0.2], np.float32)
    idx2, _, _ = oracle.select(l, 2, bias=b2, bias_mode=oracle.BIAS_PROB)
    assert list(idx2[0]) == [1, 3]
    idx3, _, _ = oracle.select(l, 3, bias=b2, bias_mode=oracle.BIAS_LOGIT)
    assert list(idx3[0]) == [1, 3, 0]


def test_select_rejects_bad_k():
    with pytest.raises(ValueError):
        oracle.select(np.zeros((1, 4)), 5)
    with pytest.raises(ValueError):
        oracle.select(np.zeros((1, 4)), 0)


# -------------------------------------------------------------------- capacity
def test_capacity_closed_forms():
    assert oracle.capacity(4096, 2, 8, 1.25) == 1280      # 1.25*4096*2/8
    assert oracle.capacity(8192, 8, 128, 1.0) == 512
    assert oracle.capacity(16384, 4, 64, 1.0) == 1024
    assert oracle.capacity(10, 1, 3, 1.0) == 4            # ceil(10/3)
    assert oracle.capacity(7, 2, 4, 0.5) == 2             # ceil(1.75)
    assert oracle.capacity(100, 2, 8, 0.0) == -1
    assert oracle.capacity(100, 2, 8, -1.0) == -1


# -------------------------------------------------------------------- dispatch
def _brute_dispatch(idx, E, cap):
    """cap: one capacity for all experts, or a list with one per expert (< 0: no limit)."""
    caps = list(cap) if hasattr(cap, "__len__") else [cap] * E
    T, K = idx.shape
    queues = [[] for _ in range(E)]
    for t in range(T):
        for k in range(K):
            queues[idx[t, k]].append((t, k))
    counts = [len(q) for q in queues]
    kept = [c if cp < 0 else min(c, cp) for c, cp in zip(counts, caps)]
    seg = [0]
    for e in range(E):
        seg.append(seg[-1] + kept[e])
    slot_of = -np.ones((T, K), np.int64)
    perm = []
    for e in range(E):
        for r, (t, k) in enumerate(queues[e][: kept[e]]):
            slot_of[t, k] = seg[e] + r
            perm.append(t * K + k)
    return counts, kept, seg, slot_of, perm


@pytest.mark.parametrize("T,E,K,cap", [(1, 1, 1, -1), (37, 5, 2, 9), (64, 8, 2, -1), (100, 16, 4, 0),
                                       (257, 7, 3, 40), (50, 4, 4, 1)])
def test_dispatch_matches_per_expert_queues(T, E, K, cap):
    rng = np.random.default_rng(T + E + K)
    # skewed: expert choices drawn without replacement with a Zipf-like prior
    pr = 1.0 / np.arange(1, E + 1) ** 1.2
    pr /= pr.sum()
    idx = np.stack([rng.choice(E, size=K, replace=False, p=pr) for _ in range(T)]).astype(np.int32)
    got = oracle.dispatch(idx, E, cap)
    counts, kept, seg, slot_of, perm = _brute_dispatch(idx, E, cap)
    assert list(got["counts"]) == counts
    assert list(got["kept"]) == kept
    assert list(got["seg_off"]) == seg
    assert (got["slot_of"] == slot_of).all()
    assert list(got["perm"]) == perm
    # invariants
    assert sum(counts) == T * K
    kept_mask = got["slot_of"] >= 0
    assert kept_mask.sum() == seg[-1]
    assert sorted(got["slot_of"][kept_mask].tolist()) == list(range(seg[-1]))


@pytest.mark.parametrize("T,E,K", [(1, 1, 1), (37, 5, 2), (257, 7, 3), (64, 16, 4)])
def test_dispatch_caps_matches_per_expert_queues(T, E, K):
    rng = np.random.default_rng(7 * T + E)
    pr = 1.0 / np.arange(1, E + 1) ** 1.2
    pr /= pr.sum()
    idx = np.stack([rng.choice(E, size=K, replace=False, p=pr) for _ in range(T)]).astype(np.int32)
    caps = rng.integers(-1, max(2, T // 2), size=E)          # includes no-limit (-1) and 0
    got = oracle.dispatch_caps(idx, E, caps)
    counts, kept, seg, slot_of, perm = _brute_dispatch(idx, E, caps.tolist())
    assert list(got["counts"]) == counts and list(got["kept"]) == kept and list(got["seg_off"]) == seg
    assert (got["slot_of"] == slot_of).all()
    assert list(got["perm"]) == perm


def test_dispatch_rejects_out_of_range_expert():
    with pytest.raises(ValueError):
        oracle.dispatch(np.array([[0, 4]], np.int32), 4, -1)


# ---------------------------------------------------------------------- SwiGLU
def test_swiglu_closed_form_single_unit():
    # d = F = 1: x = ln3, gate weight 1, up weight 2, down weight 0.5
    #   silu(ln3) = ln3 * sigmoid(ln3) = ln3 * 3/4   ->  y = 0.5 * (3/4 ln3) * (2 ln3)
    y = oracle.swiglu(np.array([LN3]), np.array([[1.0], [2.0]]), np.array([[0.5]]))
    assert y[0] == pytest.approx(0.75 * LN3 * LN3, rel=1e-15)


def test_swiglu_one_hot_weights_route_each_index():
    # Non-square d=5, F=3.  Gate row f reads x[sig[f]], up row f reads x[pi[f]]
    # with weight b[f]; output i reads h[rho[i]] with weight c[i].  Inputs take
    # values whose SiLU is known in closed form:
    #   silu(0) = 0, silu(ln3) = 3/4 ln3, silu(-ln3) = -1/4 ln3.
    d, F = 5, 3
    x = np.array([LN3, -LN3, 0.0, 2.0, -1.5])
    silu_closed = {0: LN3 * 0.75, 1: -LN3 * 0.25, 2: 0.0}
    sig = [1, 0, 2]
    pi = [3, 4, 0]
    b = [1.5, -2.0, 0.5]
    rho = [2, 0, 1, 1, 0]
    c = [1.0, 2.0, -1.0, 0.5, 3.0]
    w13 = np.zeros((2 * F, d))
    w2 = np.zeros((d, F))
    for f in range(F):
        w13[f, sig[f]] = 1.0
        w13[F + f, pi[f]] = b[f]
    for i in range(d):
        w2[i, rho[i]] = c[i]
    y = oracle.swiglu(x, w13, w2)
    for i in range(d):
        f = rho[i]
        want = c[i] * silu_closed[sig[f]] * (b[f] * x[pi[f]])
        assert y[i] == pytest.approx(want, rel=1e-14, abs=1e-15)


def test_swiglu_zero_gate_gives_zero():
    rng = np.random.default_rng(3)
    w13 = rng.normal(size=(8, 6))
    w13[:4] = 0.0
    y = oracle.swiglu(rng.normal(size=6), w13, rng.normal(size=(6, 4)))
    assert (y == 0.0).all()


# ----------------------------------------------------------------------- layer
def _rand_layer(rng, T, d, E, F, Ns=0):
    x = rng.normal(size=(T, d))
    w13 = rng.normal(size=(E, 2 * F, d)) / math.sqrt(d)
    w2 = rng.normal(size=(E, d, F)) / math.sqrt(F)
    sh = (rng.normal(size=(Ns, 2 * F, d)) / math.sqrt(d), rng.normal(size=(Ns, d, F)) / math.sqrt(F)) if Ns else (None, None)
    return x, w13, w2, sh


def test_layer_single_expert_top1_is_dense_swiglu():
    rng = np.random.default_rng(4)
    T, d, F = 9, 12, 10
    x, w13, w2, _ = _rand_layer(rng, T, d, 1, F)
    l = rng.normal(size=(T, 1))
    idx, w, _ = oracle.select(l, 1)
    assert (w == 1.0).all()
    disp = oracle.dispatch(idx, 1, oracle.capacity(T, 1, 1, 0.0))
    y = oracle.layer_rows(x, w13, w2, idx, w, disp["slot_of"])
    for t in range(T):
        assert np.allclose(y[t], oracle.swiglu(x[t], w13[0], w2[0]), rtol=0, atol=1e-13)


def test_layer_shared_experts_equal_one_concatenated_swiglu():
    # sum_s W2_s (silu(G_s x) * U_s x) == [W2_0 | W2_1 | ..] (silu([G_0;G_1;..] x) * [U_0;U_1;..] x)
    rng = np.random.default_rng(5)
    T, d, E, F, Ns = 4, 8, 3, 5, 3
    x, w13, w2, (w13s, w2s) = _rand_layer(rng, T, d, E, F, Ns)
    idx = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1))
    slot_none = -np.ones((T, 1), np.int32)        # every routed pair dropped
    y = oracle.layer_rows(x, w13, w2, idx, w, slot_none, w13_shared=w13s, w2_shared=w2s)
    gate = np.concatenate([w13s[s, :F] for s in range(Ns)])
    up = np.concatenate([w13s[s, F:] for s in range(Ns)])
    down = np.concatenate([w2s[s] for s in range(Ns)], axis=1)
    big13 = np.concatenate([gate, up])
    for t in range(T):
        assert np.allclose(y[t], oracle.swiglu(x[t], big13, down), rtol=0, atol=1e-12)


def test_layer_is_gate_weighted_sum_and_drops_contribute_nothing():
    rng = np.random.default_rng(6)
    T, d, E, F = 6, 10, 4, 7
    x, w13, w2, _ = _rand_layer(rng, T, d, E, F)
    idx = np.array([[0, 1], [1, 2], [2, 3], [3, 0], [0, 2], [1, 3]], np.int32)
    w = rng.uniform(0.1, 0.9, size=(T, 2))
    disp = oracle.dispatch(idx, E, 2)       # every expert keeps its first 2 tokens
    y = oracle.layer_rows(x, w13, w2, idx, w, disp["slot_of"])
    for t in range(T):
        want = np.zeros(d)
        for k in range(2):
            if disp["slot_of"][t, k] >= 0:
                want += w[t, k] * oracle.swiglu(x[t], w13[idx[t, k]], w2[idx[t, k]])
        assert np.allclose(y[t], want, rtol=0, atol=1e-13)
    # tokens 4 and 5 arrive after each of their experts is full
    assert (disp["slot_of"][4:] == -1).all()
    assert (y[4:] == 0.0).all()


def _pipeline(x, wg, w13, w2, K, C):
    T, E = x.shape[0], wg.shape[0]
    idx, w, _ = oracle.select(oracle.gate_logits(x, wg), K)
    disp = oracle.dispatch(idx, E, oracle.capacity(T, K, E, C))
    return oracle.layer_rows(x, w13, w2, idx, w, disp["slot_of"]), idx, disp


def test_layer_is_unchanged_by_relabelling_the_experts():
    # Expert j of the relabelled layer is expert pi[j] of the original (its gate
    # row and weights move together): every token picks the same experts under
    # new names, in the same order, each expert queues the same tokens, so the
    # output -- drops under the capacity included -- is the same up to the
    # rounding of sums over experts taken in another order (a slip in an expert
    # index changes it by O(1)).
    rng = np.random.default_rng(21)
    T, d, E, K, F = 40, 12, 6, 2, 9
    x, w13, w2, _ = _rand_layer(rng, T, d, E, F)
    wg = rng.normal(size=(E, d)) / math.sqrt(d)
    y, idx, disp = _pipeline(x, wg, w13, w2, K, 0.75)
    assert int(disp["seg_off"][-1]) < T * K                    # the capacity drops pairs
    pi = rng.permutation(E)
    inv = np.argsort(pi)
    y2, idx2, disp2 = _pipeline(x, wg[pi], w13[pi], w2[pi], K, 0.75)
    assert (idx2 == inv[idx]).all()
    assert ((disp2["slot_of"] >= 0) == (disp["slot_of"] >= 0)).all()
    assert np.max(np.abs(y2 - y)) <= 1e-14 * np.max(np.abs(y))


def test_layer_without_capacity_permutes_with_its_tokens():
    # With no capacity limit nothing depends on the order of arrival: output row
    # i of the permuted batch is output row sigma[i] of the original.
    rng = np.random.default_rng(22)
    T, d, E, K, F = 33, 10, 5, 3, 8
    x, w13, w2, _ = _rand_layer(rng, T, d, E, F)
    wg = rng.normal(size=(E, d)) / math.sqrt(d)
    y, _, disp = _pipeline(x, wg, w13, w2, K, 0.0)
    assert int(disp["seg_off"][-1]) == T * K
    sigma = rng.permutation(T)
    y2, _, _ = _pipeline(x[sigma], wg, w13, w2, K, 0.0)
    assert np.array_equal(y2, y[sigma])


def test_layer_rows_subset_matches_full():
    rng = np.random.default_rng(7)
    T, d, E, F = 11, 8, 4, 6
    x, w13, w2, _ = _rand_layer(rng, T, d, E, F)
    idx, w, _ = oracle.select(rng.normal(size=(T, E)), 2)
    disp = oracle.dispatch(idx, E, -1)
    full = oracle.layer_rows(x, w13, w2, idx, w, disp["slot_of"])
    rows = np.array([10, 0, 5])
    sub = oracle.layer_rows(x, w13, w2, idx, w, disp["slot_of"], rows=rows)
    assert (sub == full[rows]).all()


def test_combine_of_grouped_expert_outputs_equals_layer():
    # Run every kept (t,k) row through its expert, lay the results out in slot
    # order, combine: must equal layer_rows, which evaluates per token.
    rng = np.random.default_rng(9)
    T, d, E, F, Ns = 13, 8, 4, 6, 2
    x, w13, w2, (w13s, w2s) = _rand_layer(rng, T, d, E, F, Ns)
    idx, w, _ = oracle.select(rng.normal(size=(T, E)), 2)
    disp = oracle.dispatch(idx, E, 5)
    S = int(disp["seg_off"][-1])
    y_perm = np.zeros((S, d))
    for s_ in range(S):
        t, k = divmod(int(disp["perm"][s_]), 2)
        y_perm[s_] = oracle.swiglu(x[t], w13[idx[t, k]], w2[idx[t, k]])
    y_sh = np.stack([sum(oracle.swiglu(x[t], w13s[s], w2s[s]) for s in range(Ns)) for t in range(T)])
    y = oracle.combine(y_perm, disp["slot_of"], w, y_sh)
    want = oracle.layer_rows(x, w13, w2, idx, w, disp["slot_of"], w13_shared=w13s, w2_shared=w2s)
    assert np.allclose(y, want, rtol=0, atol=1e-13)


def test_combine_hand_example():
    y_perm = np.array([[1.0, 2.0], [10.0, 20.0], [100.0, 200.0]])
    slot_of = np.array([[2, -1], [0, 1]], np.int32)
    w = np.array([[0.5, 0.5], [0.25, 0.75]])
    y = oracle.combine(y_perm, slot_of, w, y_shared=np.array([[1.0, 1.0], [0.0, 0.0]]))
    assert y.tolist() == [[51.0, 101.0], [7.75, 15.5]]
    assert oracle.combine(y_perm, slot_of, w).tolist() == [[50.0, 100.0], [7.75, 15.5]]


# --------------------------------------------------------------- balance stats
def test_balance_uniform_routing_gives_exactly_alpha():
    g = golden("balance_alpha.json")
    for E, K, T in [(8, 2, 64), (128, 8, 256), (64, 4, 128)]:
        # all-equal logits: P_e = 1/E exactly; round-robin routing: f_e = 1/E
        p = oracle.softmax(np.zeros((T, E)))
        idx = np.array([[(t * K + k) % E for k in range(K)] for t in range(T)], np.int32)
        counts = oracle.dispatch(idx, E, -1)["counts"]
        f, P, loss = oracle.balance(counts, p, K, alpha=g["alpha"])
        assert (P == 1.0 / E).all() and (f == 1.0 / E).all()
        assert loss == g["uniform_loss"]


def test_balance_uniform_load_any_probabilities_gives_alpha():
    rng = np.random.default_rng(8)
    E, K, T = 16, 2, 64
    p = oracle.softmax(rng.normal(size=(T, E)) * 4)
    counts = np.full(E, T * K // E, np.int32)
    _, _, loss = oracle.balance(counts, p, K, alpha=0.01)
    assert loss == pytest.approx(0.01, rel=1e-14)


def test_balance_hand_example():
    # E=2, K=1, T=4: counts [3, 1] -> f = [3/4, 1/4]; p rows given directly
    p = np.array([[0.5, 0.5], [0.9, 0.1], [0.7, 0.3], [0.1, 0.9]])
    f, P, loss = oracle.balance(np.array([3, 1], np.int32), p, 1, alpha=0.01)
    assert list(f) == [0.75, 0.25]
    assert P == pytest.approx([0.55, 0.45], abs=1e-15)
    assert loss == pytest.approx(0.01 * 2 * (0.75 * 0.55 + 0.25 * 0.45), rel=1e-14)


# ----------------------------------------------------------- z-loss / utilisation
def test_router_zloss_closed_form():
    assert oracle.router_zloss(np.zeros((5, 4))) == pytest.approx(math.log(4) ** 2, rel=1e-15)
    assert oracle.router_zloss(np.full((2, 8), 1.5)) == pytest.approx((1.5 + math.log(8)) ** 2, rel=1e-15)


def test_utilization_uniform_is_max_entropy_golden():
    g = golden("utilization_max_entropy.json")
    E = g["n_experts"]
    u = oracle.utilization(np.full(E, 40, np.int32), np.full(E, 40, np.int32))
    assert u["entropy_bits"] == pytest.approx(g["max_bits"], abs=1e-12)
    assert u["cv"] == 0.0 and u["drop_rate"] == 0.0
    assert u["n_below_half"] == 0 and u["n_above_double"] == 0


def test_utilization_hand_example():
    counts = np.array([8, 0, 0, 0], np.int32)
    u = oracle.utilization(counts, np.array([4, 0, 0, 0], np.int32))
    assert u["entropy_bits"] == 0.0
    assert u["drop_rate"] == 0.5
    assert u["cv"] == pytest.approx(math.sqrt(3.0), rel=1e-15)   # std 2*sqrt3, mean 2
    assert u["n_below_half"] == 3 and u["n_above_double"] == 1
    u2 = oracle.utilization(np.array([1, 1, 2], np.int32), np.array([1, 1, 2], np.int32))
    assert u2["entropy_bits"] == pytest.approx(1.5, abs=1e-15)


def test_flops_ratio_golden_compute_budget():
    g = golden("compute_budget_ratio.json")
    E, K, Ns, T = g["N_E"], g["K"], g["N_shared"], 96
    _, expert, ratio = oracle.flops(T, 7168, E, 2048, Ns, kept_pairs=T * K)
    assert ratio == g["ratio_numerator"] / g["ratio_denominator"]
    assert round(100 * ratio, 1) == g["printed_percent"]
    assert expert == 6.0 * 7168 * 2048 * (K + Ns) * T


# ----------------------------------------------------- bias update (Zen-Max §2.3)
def test_bias_update_sign_hand_example():
    # E=4, T*K=8: target load 2.  Loads 4, 2, 1, 1: overloaded, balanced, under, under.
    b = oracle.bias_update([4, 2, 1, 1], 8, [0.0, 0.0, 0.0, 0.0], 0.125, oracle.BIAS_UPDATE_SIGN)
    assert b.tolist() == [-0.125, 0.0, 0.125, 0.125]
    b2 = oracle.bias_update([4, 2, 1, 1], 8, b, 0.125, oracle.BIAS_UPDATE_SIGN)
    assert b2.tolist() == [-0.25, 0.0, 0.25, 0.25]


def test_bias_update_proportional_hand_example_and_zero_sum():
    # relative deviation (target - load) / target = (2 - c) / 2
    b = oracle.bias_update([4, 2, 1, 1], 8, [1.0, 1.0, 1.0, 1.0], 0.5, oracle.BIAS_UPDATE_PROPORTIONAL)
    assert b.tolist() == [0.5, 1.0, 1.25, 1.25]
    rng = np.random.default_rng(3)
    for E in (3, 8, 64):
        counts = rng.multinomial(1000, np.ones(E) / E).astype(np.int32)
        d = oracle.bias_update(counts, 1000, np.zeros(E), 1.0, oracle.BIAS_UPDATE_PROPORTIONAL)
        # the steps are E*(target - load)/TK: they sum to zero up to one rounding each
        assert abs(float(np.sum(d.astype(np.float64)))) <= E * 2.0 ** -23


def test_bias_update_balanced_load_leaves_bias_unchanged():
    for mode in (oracle.BIAS_UPDATE_SIGN, oracle.BIAS_UPDATE_PROPORTIONAL):
        b0 = np.array([0.3, -0.2, 0.0, 1e-3], np.float32)
        assert (oracle.bias_update([5, 5, 5, 5], 20, b0, 0.01, mode) == b0).all()


def test_bias_update_closes_the_loop_on_a_fixed_router():
    # Fixed probabilities favouring expert 0; top-1 selection on p + b.  Repeated
    # updates must pull the selection towards a balanced load (the page's purpose).
    rng = np.random.default_rng(11)
    T, E, K = 512, 4, 1
    logits = rng.normal(size=(T, E)) + np.array([1.0, 0.0, 0.0, 0.0])
    b = np.zeros(E, np.float32)
    first = None
    for step in range(200):
        idx, _, _ = oracle.select(logits, K, bias=b)
        counts = np.bincount(idx.ravel(), minlength=E).astype(np.int32)
        if first is None:
            first = counts.max() - counts.min()
        b = oracle.bias_update(counts, T * K, b, 0.002, oracle.BIAS_UPDATE_SIGN)
    assert first > 150 and counts.max() - counts.min() < first / 4
    assert b[0] < 0 < min(b[1:])


# ----------------------------------------- adaptive capacity (Zen MoDE §5.3)
def test_adaptive_capacity_hand_example():
    # T=8, K=1, E=4, one batch with loads 4, 2, 1, 1: fbar = .5, .25, .125, .125
    # C_e = 1 + 2 (fbar - 1/4) = 1.5, 1, .75, .75; cap = ceil(C_e * 8 / 4) = 3, 2, 2, 2
    caps = oracle.adaptive_capacity(8, 1, [[4, 2, 1, 1]], 1.0, 2.0)
    assert caps.tolist() == [3, 2, 2, 2]


def test_adaptive_capacity_reduces_to_uniform_capacity():
    # gamma = 0, or a window whose mean load is uniform: every expert gets ceil(C T K / E)
    hist = np.array([[1100, 990, 1010, 996, 1000, 1024, 1000, 1072]], np.int32)   # sums to 8192
    assert oracle.adaptive_capacity(4096, 2, hist, 1.25, 0.0).tolist() == [1280] * 8
    flat = np.array([[1024] * 8, [1024] * 8], np.int32)
    assert oracle.adaptive_capacity(4096, 2, flat, 1.25, 3.0).tolist() == [1280] * 8


def test_adaptive_capacity_window_mean_and_clamps():
    # two batches that average to a uniform load: the window sees no skew
    hist = [[4, 2, 1, 1], [0, 2, 3, 3]]
    assert oracle.adaptive_capacity(8, 1, hist, 1.0, 2.0).tolist() == [2, 2, 2, 2]
    # everything on expert 0: C = 1 + 5 (1 - 1/4) = 4.75 -> ceil(9.5) = 10 -> clamped to T = 8;
    # the others: 1 - 5/4 < 0 -> 0
    assert oracle.adaptive_capacity(8, 1, [[8, 0, 0, 0]], 1.0, 5.0).tolist() == [8, 0, 0, 0]


def test_adaptive_capacity_monotone_in_load():
    rng = np.random.default_rng(5)
    E = 16
    hist = rng.multinomial(4096, rng.dirichlet(np.ones(E)), size=3).astype(np.int32)
    caps = oracle.adaptive_capacity(2048, 2, hist, 1.0, 4.0)
    load = hist.sum(0)
    order = np.argsort(load, kind="stable")
    assert (np.diff(caps[order]) >= 0).all()
    # under-used experts lose budget, over-used gain it (page: prevents drops under skew)
    base = oracle.capacity(2048, 2, E, 1.0)
    assert (caps[load < load.mean()] <= base).all() and (caps[load > load.mean()] >= base).all()


# ---------------------------------------------- layer backward (training)
def _fd_problem(seed=0, T=6, d=5, E=4, K=2, F=3, Ns=1, cap=3):
    rng = np.random.default_rng(seed)
    P = dict(x=rng.normal(size=(T, d)), wg=rng.normal(size=(E, d)) * 0.7, off=rng.normal(size=E).astype(np.float32),
             w13=rng.normal(size=(E, 2 * F, d)) * 0.5, w2=rng.normal(size=(E, d, F)) * 0.5,
             w13s=rng.normal(size=(Ns, 2 * F, d)) * 0.5, w2s=rng.normal(size=(Ns, d, F)) * 0.5)
    R = rng.normal(size=(T, d))
    return P, R, dict(T=T, d=d, E=E, K=K, F=F, Ns=Ns, cap=cap)


def _objective(P, R, c, idx_fixed, slot_fixed, counts_fixed, c_bal, c_z, alpha=0.01):
    """J = sum(R * y) + c_bal * L_balance + c_z * L_z through the oracle's own forward,
    with the routing (chosen experts, capacity cut, counts) held fixed."""
    logits = oracle.gate_logits(P["x"], P["wg"], P["off"])
    idx, w, p = oracle.select(logits, c["K"])
    assert (idx == idx_fixed).all(), "perturbation changed the routing"
    y = oracle.layer_rows(P["x"], P["w13"], P["w2"], idx, w, slot_fixed,
                          w13_shared=P["w13s"] if c["Ns"] else None, w2_shared=P["w2s"] if c["Ns"] else None)
    _, _, loss = oracle.balance(counts_fixed, p, c["K"], alpha)
    return float(np.sum(R * y)) + c_bal * loss + c_z * oracle.router_zloss(logits)


@pytest.mark.parametrize("seed,c_bal,c_z,cap", [(0, 1.0, 0.0, 3), (1, 0.7, 0.3, 2), (2, 0.0, 1.0, -1)])
def test_layer_backward_matches_finite_differences(seed, c_bal, c_z, cap):
    P, R, c = _fd_problem(seed, cap=cap)
    alpha = 0.01
    logits = oracle.gate_logits(P["x"], P["wg"], P["off"])
    idx, w, p = oracle.select(logits, c["K"])
    disp = oracle.dispatch(idx, c["E"], cap)
    assert cap < 0 or (disp["slot_of"] < 0).any() or cap >= c["T"]
    g = oracle.layer_backward(P["x"], P["wg"], P["w13"], P["w2"], logits, idx, w, disp["slot_of"], disp["counts"],
                              alpha, R, c_bal, c_z, P["w13s"], P["w2s"])
    h = 1e-6
    names = {"x": "dx", "wg": "dwg", "w13": "dw13", "w2": "dw2", "w13s": "dw13_shared", "w2s": "dw2_shared"}
    for name, gname in names.items():
        arr = P[name]
        fd = np.empty_like(arr)
        for i in np.ndindex(arr.shape):
            keep = arr[i]
            arr[i] = keep + h
            jp = _objective(P, R, c, idx, disp["slot_of"], disp["counts"], c_bal, c_z, alpha)
            arr[i] = keep - h
            jm = _objective(P, R, c, idx, disp["slot_of"], disp["counts"], c_bal, c_z, alpha)
            arr[i] = keep
            fd[i] = (jp - jm) / (2 * h)
        err = np.max(np.abs(fd - g[gname]))
        assert err <= 1e-6 * max(1.0, float(np.max(np.abs(fd)))), (name, err)
    # the offset (a float32 input) enters like a logit shared by all tokens; steps of
    # 2^-12 are exact in float32 at these magnitudes, so the difference quotient is exact
    fdo = np.empty(c["E"])
    hs = np.float32(2.0 ** -12)
    for e in range(c["E"]):
        P2 = dict(P)
        o = P["off"].copy(); o[e] += hs
        P2["off"] = o
        jp = _objective(P2, R, c, idx, disp["slot_of"], disp["counts"], c_bal, c_z, alpha)
        o = P["off"].copy(); o[e] -= hs
        P2["off"] = o
        jm = _objective(P2, R, c, idx, disp["slot_of"], disp["counts"], c_bal, c_z, alpha)
        fdo[e] = (jp - jm) / (2.0 * float(hs))
    assert np.max(np.abs(fdo - g["doff"])) <= 1e-5 * max(1.0, float(np.max(np.abs(fdo))))


def test_layer_backward_offset_gradient_sums_to_zero_without_zloss():
    # the gate-weight and balance terms are softmax Jacobians: each token's dl sums to 0
    P, R, c = _fd_problem(5, T=9, E=6, K=3)
    logits = oracle.gate_logits(P["x"], P["wg"], P["off"])
    idx, w, p = oracle.select(logits, c["K"])
    disp = oracle.dispatch(idx, c["E"], -1)
    g = oracle.layer_backward(P["x"], P["wg"], P["w13"], P["w2"], logits, idx, w, disp["slot_of"], disp["counts"],
                              0.01, R, 1.0, 0.0, P["w13s"], P["w2s"])
    assert abs(float(np.sum(g["doff"]))) <= 1e-12
    g2 = oracle.layer_backward(P["x"], P["wg"], P["w13"], P["w2"], logits, idx, w, disp["slot_of"], disp["counts"],
                               0.01, R, 1.0, 1.0, P["w13s"], P["w2s"])
    # with the z-loss: sum_e dl_e = (2/T) lse_t per token
    lse = np.log(np.sum(np.exp(logits - logits.max(1, keepdims=True)), 1)) + logits.max(1)
    assert abs(float(np.sum(g2["doff"])) - float(np.sum(2.0 / c["T"] * lse))) <= 1e-12 * max(1.0, float(np.sum(np.abs(lse))))


def test_layer_backward_dropped_pairs_give_their_expert_no_gradient():
    P, R, c = _fd_problem(3, T=8, E=4, K=2, cap=1)
    logits = oracle.gate_logits(P["x"], P["wg"], P["off"])
    idx, w, p = oracle.select(logits, c["K"])
    disp = oracle.dispatch(idx, c["E"], 1)
    g = oracle.layer_backward(P["x"], P["wg"], P["w13"], P["w2"], logits, idx, w, disp["slot_of"], disp["counts"],
                              0.01, R, 0.0, 0.0, P["w13s"], P["w2s"])
    for e in range(c["E"]):
        if disp["kept"][e] == 0:
            assert not g["dw13"][e].any() and not g["dw2"][e].any()


def test_layer_backward_logit_gradient_matches_finite_differences():
    P, R, c = _fd_problem(7, T=5, E=5, K=2, cap=2)
    alpha, c_bal, c_z = 0.01, 0.9, 0.4
    logits = oracle.gate_logits(P["x"], P["wg"], P["off"])
    idx, w, p = oracle.select(logits, c["K"])
    disp = oracle.dispatch(idx, c["E"], c["cap"])
    g = oracle.layer_backward(P["x"], P["wg"], P["w13"], P["w2"], logits, idx, w, disp["slot_of"], disp["counts"],
                              alpha, R, c_bal, c_z, P["w13s"], P["w2s"])

    def J(l):
        i2, w2, p2 = oracle.select(l, c["K"])
        assert (i2 == idx).all()
        y = oracle.layer_rows(P["x"], P["w13"], P["w2"], i2, w2, disp["slot_of"], w13_shared=P["w13s"],
                              w2_shared=P["w2s"])
        _, _, loss = oracle.balance(disp["counts"], p2, c["K"], alpha)
        return float(np.sum(R * y)) + c_bal * loss + c_z * oracle.router_zloss(l)

    fd = np.empty_like(logits)
    for i in np.ndindex(logits.shape):
        lp = logits.copy(); lp[i] += 1e-6
        lm = logits.copy(); lm[i] -= 1e-6
        fd[i] = (J(lp) - J(lm)) / 2e-6
    assert np.max(np.abs(fd - g["dlogits"])) <= 1e-6 * max(1.0, float(np.max(np.abs(fd))))
    assert np.allclose(g["dlogits"].sum(0), g["doff"], rtol=0, atol=1e-12)


def test_openmp_build_gives_the_same_bits():
    """The -fopenmp build of the oracle (the CPU baseline's second figure)
    splits the outer loops of the gate logits and the layer rows over threads;
    each output is still one thread's sum in the same order, so every value is
    the same bits as the single-thread build's (shared experts, drops and a
    bias included)."""
    rng = np.random.default_rng(7)
    T, d, E, K, F, Ns = 37, 48, 6, 2, 40, 1
    bf = lambda a: (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    x = bf(rng.normal(size=(T, d)))
    wg = bf(rng.normal(size=(E, d)) / np.sqrt(d))
    w13 = bf(rng.normal(size=(E, 2 * F, d)) / np.sqrt(d))
    w2 = bf(rng.normal(size=(E, d, F)) / np.sqrt(F))
    w13s = bf(rng.normal(size=(Ns, 2 * F, d)) / np.sqrt(d))
    w2s = bf(rng.normal(size=(Ns, d, F)) / np.sqrt(F))
    bias = rng.uniform(-0.05, 0.05, size=E).astype(np.float32)
    offset = rng.normal(size=E).astype(np.float32)

    def run():
        l = oracle.gate_logits(x, wg, offset)
        idx, w, p = oracle.select(l, K, bias=bias)
        disp = oracle.dispatch(idx, E, 9)
        y = oracle.layer_rows(x, w13, w2, idx, w, disp["slot_of"], w13_shared=w13s, w2_shared=w2s)
        return l, idx, w, disp["slot_of"], y

    seq = run()
    try:
        n = oracle.set_threads(4)
        omp = run()
    finally:
        assert oracle.set_threads(1) == 1
    assert n == 4
    assert (seq[3] < 0).any()          # some pairs dropped
    for a, b in zip(seq, omp):
        assert a.dtype == b.dtype and np.array_equal(a.view(np.uint8), b.view(np.uint8))
