"""GPU parity against the float64 oracle, stage by stage and end to end, on
sizes the oracle finishes in seconds (several tiles, ragged tails, edge cases).

Bars: routing (expert indices, counts, kept, offsets, slots, permutation,
dropped set) bit-exact when both sides get the same float32 logits; gate
weights within 1e-6; layer outputs within max relative error 2e-2 (BF16) or
1e-4 (FP32), where max relative error = max|y - y_ref| / max|y_ref|.
Every call goes through the C ABI (libmoe_b200.so)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import (dev, generate, given_logits, host_np, oracle_layer, oracle_routing, problem, rel_err,
                     sample_rows, tol)
from sparse_mixture_experts_04_b200 import MoeLayer, api
from sparse_mixture_experts_04_b200.synth import CONFIGS, MoeConfig

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny_fp32": CONFIGS["tiny_fp32"],
    "mini_mixtral": MoeConfig("mini_mixtral", T=777, d_model=512, n_experts=8, top_k=2, d_ff=384, n_shared=0,
                              capacity_factor=1.25, dtype="bf16", seed=11),
    "mini_zen": MoeConfig("mini_zen", T=500, d_model=256, n_experts=128, top_k=8, d_ff=128, n_shared=4,
                          capacity_factor=1.0, dtype="bf16", seed=12, bias_range=0.1),
    "mini_skewed": MoeConfig("mini_skewed", T=1000, d_model=256, n_experts=64, top_k=4, d_ff=200, n_shared=0,
                             capacity_factor=1.0, dtype="bf16", seed=13, zipf_s=1.2),
    "mini_decode": MoeConfig("mini_decode", T=32, d_model=512, n_experts=128, top_k=8, d_ff=256, n_shared=1,
                             capacity_factor=0.0, dtype="bf16", seed=14),
    "ragged_bf16": MoeConfig("ragged_bf16", T=300, d_model=520, n_experts=7, top_k=3, d_ff=200, n_shared=2,
                             capacity_factor=0.9, dtype="bf16", seed=15, bias_range=0.05),
    "ragged_f32": MoeConfig("ragged_f32", T=100, d_model=72, n_experts=5, top_k=2, d_ff=40, n_shared=1,
                            capacity_factor=1.0, dtype="f32", seed=16, x_std=0.5),
    "single_expert": MoeConfig("single_expert", T=1, d_model=64, n_experts=1, top_k=1, d_ff=64, n_shared=0,
                               capacity_factor=0.0, dtype="bf16", seed=17),
    "k_equals_e": MoeConfig("k_equals_e", T=129, d_model=128, n_experts=4, top_k=4, d_ff=136, n_shared=0,
                            capacity_factor=1.0, dtype="bf16", seed=18),
    "tiny_capacity": MoeConfig("tiny_capacity", T=257, d_model=64, n_experts=16, top_k=2, d_ff=64, n_shared=1,
                               capacity_factor=0.05, dtype="bf16", seed=19),
    "wide_e256": MoeConfig("wide_e256", T=200, d_model=128, n_experts=256, top_k=6, d_ff=64, n_shared=0,
                           capacity_factor=2.0, dtype="bf16", seed=20, bias_range=0.01),
    # the largest top-K of this build (32, with a bias on p: K + 1 ranking rounds exceed the warp)
    "max_k32": MoeConfig("max_k32", T=96, d_model=128, n_experts=256, top_k=32, d_ff=64, n_shared=1,
                         capacity_factor=1.0, dtype="bf16", seed=23, bias_range=0.01),
}


def _inputs(name):
    return generate(SMALL[name])


_cache = {}


def inputs(name):
    if name not in _cache:
        _cache[name] = _inputs(name)
    return _cache[name]


# ------------------------------------------------------------------- routing
def _route_given(cfg, logits32, sel_bias, flags=api.FLAG_LOGITS_GIVEN):
    prob = problem(cfg, flags)
    ws = api.alloc_workspace(prob)
    T, E, K = cfg.T, cfg.n_experts, cfg.top_k
    lg = dev(logits32)
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    stats = torch.empty(2 * E + 1, dtype=torch.float32, device="cuda")
    api.reset_device_status(ws)
    api.moe_route(prob, None, None, None, dev(sel_bias), lg, idx, w, stats, ws)
    assert api.read_device_status(ws) == 0
    return idx.cpu().numpy(), w.cpu().numpy(), stats.cpu().numpy()


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("bias_on_logit", [False, True])
def test_route_from_given_logits_is_bit_exact(name, bias_on_logit):
    cfg = SMALL[name]
    inp = inputs(name)
    if bias_on_logit and inp["sel_bias"] is None:
        pytest.skip("no selection bias in this workload")
    flags = api.FLAG_LOGITS_GIVEN | (api.FLAG_BIAS_LOGIT if bias_on_logit else 0)
    logits32 = given_logits(cfg)
    ref = oracle_routing(cfg, logits32.astype(np.float64), inp["sel_bias"], flags)
    idx, w, stats = _route_given(cfg, logits32, inp["sel_bias"], flags)
    assert (idx == ref["idx"]).all()
    assert np.max(np.abs(w - ref["w"])) <= 1e-6
    assert np.allclose(w.sum(1), 1.0, atol=1e-6)
    E = cfg.n_experts
    assert (stats[:E] == ref["f"].astype(np.float32)).all()
    assert np.max(np.abs(stats[E:2 * E] - ref["P"])) <= 1e-6
    assert abs(stats[2 * E] - ref["loss"]) <= 1e-6 * max(1.0, abs(ref["loss"]))


@pytest.mark.parametrize("E,K", [(8, 2), (64, 4), (128, 8), (7, 7)])
def test_route_ties_go_to_lower_index(E, K):
    cfg = MoeConfig("ties", T=70, d_model=64, n_experts=E, top_k=K, d_ff=64, n_shared=0, capacity_factor=0.0,
                    dtype="bf16", seed=0)
    rng = np.random.default_rng(E)
    logits32 = rng.integers(-2, 3, size=(70, E)).astype(np.float32)   # many exact ties
    logits32[:5] = 0.0                                                 # all-equal rows
    ref = oracle_routing(cfg, logits32.astype(np.float64), None)
    idx, w, _ = _route_given(cfg, logits32, None)
    assert (idx == ref["idx"]).all()
    assert (idx[:5] == np.arange(K)).all()
    assert np.max(np.abs(w - ref["w"])) <= 1e-6


def test_route_extreme_logits():
    cfg = MoeConfig("extreme", T=64, d_model=64, n_experts=16, top_k=3, d_ff=64, n_shared=0, capacity_factor=0.0,
                    dtype="bf16", seed=0, bias_range=0.2)
    rng = np.random.default_rng(3)
    logits32 = (rng.normal(size=(64, 16)) * 40).astype(np.float32)
    bias = rng.uniform(-0.2, 0.2, 16).astype(np.float32)
    ref = oracle_routing(cfg, logits32.astype(np.float64), bias)
    idx, w, _ = _route_given(cfg, logits32, bias)
    assert (idx == ref["idx"]).all()
    assert np.max(np.abs(w - ref["w"])) <= 1e-6


@pytest.mark.parametrize("name", list(SMALL))
def test_gate_logits_match_oracle(name):
    cfg = SMALL[name]
    inp = inputs(name)
    prob = problem(cfg)
    ws = api.alloc_workspace(prob)
    T, E, K = cfg.T, cfg.n_experts, cfg.top_k
    lg = torch.empty((T, E), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    api.moe_route(prob, dev(inp["x"]), dev(inp["w_gate"]), dev(inp["logit_offset"]), dev(inp["sel_bias"]), lg,
                  idx, w, None, ws)
    got = lg.cpu().numpy().astype(np.float64)
    want = oracle.gate_logits(host_np(inp["x"]), host_np(inp["w_gate"]), inp["logit_offset"])
    bound = (1e-5 if cfg.dtype == "f32" else 1e-3) * max(1.0, float(np.max(np.abs(want))))
    assert np.max(np.abs(got - want)) <= bound


# ------------------------------------------------------------------ dispatch
@pytest.mark.parametrize("name", list(SMALL))
def test_dispatch_is_bit_exact(name):
    cfg = SMALL[name]
    inp = inputs(name)
    ref = oracle_routing(cfg, given_logits(cfg).astype(np.float64), inp["sel_bias"])
    prob = problem(cfg)
    ws = api.alloc_workspace(prob)
    E, T, K = cfg.n_experts, cfg.T, cfg.top_k
    R = max(api.max_rows(prob), 1)
    i32 = dict(dtype=torch.int32, device="cuda")
    counts, kept, seg = torch.empty(E, **i32), torch.empty(E, **i32), torch.empty(E + 1, **i32)
    slot_of = torch.empty((T, K), **i32)
    perm = torch.full((R,), -7, **i32)
    x = dev(inp["x"])
    x_perm = torch.zeros((R, cfg.d_model), dtype=x.dtype, device="cuda")
    api.reset_device_status(ws)
    api.moe_dispatch(prob, dev(ref["idx"]), x, counts, kept, seg, slot_of, perm, x_perm, ws)
    assert api.read_device_status(ws) == 0
    assert (counts.cpu().numpy() == ref["counts"]).all()
    assert (kept.cpu().numpy() == ref["kept"]).all()
    assert (seg.cpu().numpy() == ref["seg_off"]).all()
    assert (slot_of.cpu().numpy() == ref["slot_of"]).all()
    S = int(ref["seg_off"][-1])
    assert (perm.cpu().numpy()[:S] == ref["perm"]).all()
    assert (perm.cpu().numpy()[S:] == -7).all()            # untouched past the kept total
    src = torch.as_tensor(ref["perm"].astype(np.int64) // K)
    assert torch.equal(x_perm[:S].cpu(), inp["x"][src])      # gathered rows are bit copies


def test_dispatch_flags_out_of_range_expert_without_faulting():
    cfg = MoeConfig("bad", T=40, d_model=64, n_experts=8, top_k=2, d_ff=64, n_shared=0, capacity_factor=0.0,
                    dtype="bf16", seed=0)
    prob = problem(cfg)
    ws = api.alloc_workspace(prob)
    idx = np.tile(np.array([[0, 1]], np.int32), (40, 1))
    idx[5, 1] = 9      # outside [0, E): skipped by the kernels' own bounds checks
    idx[7, 0] = -3
    i32 = dict(dtype=torch.int32, device="cuda")
    counts, kept, seg = torch.empty(8, **i32), torch.empty(8, **i32), torch.empty(9, **i32)
    slot_of = torch.empty((40, 2), **i32)
    perm = torch.empty(80, **i32)
    api.reset_device_status(ws)
    api.moe_dispatch(prob, dev(idx), None, counts, kept, seg, slot_of, perm, None, ws)
    bits = api.read_device_status(ws)
    assert bits & 0x1
    s = slot_of.cpu().numpy()
    assert s[5, 1] == -1 and s[7, 0] == -1
    assert counts.cpu().numpy()[0] == 39 and counts.cpu().numpy()[1] == 39


@pytest.mark.parametrize("T,E,K", [(32768, 256, 4), (32769, 256, 4), (65536, 64, 4), (65537, 64, 4)])
def test_layer_routing_and_stats_on_both_sides_of_the_fused_scan_limit(T, E, K):
    """Dispatch ranks with one fused scan+rank kernel while ceil(T/256)^2 * E
    <= 2^22 and with a scan kernel then a rank kernel above; each pair of
    cases sits on the two sides of that limit.  Routing bit-exact and the
    balance / extended statistics against the oracle, through the layer."""
    cfg = MoeConfig(f"limit_{T}_{E}", T=T, d_model=64, n_experts=E, top_k=K, d_ff=64, n_shared=0,
                    capacity_factor=1.0, dtype="bf16", seed=21, zipf_s=1.1)
    inp = generate(cfg)
    logits32 = given_logits(cfg)
    ref = oracle_routing(cfg, logits32.astype(np.float64), inp["sel_bias"])
    layer = MoeLayer.from_inputs(inp, flags=api.FLAG_LOGITS_GIVEN | api.FLAG_EXTENDED_STATS)
    layer.routing["logits"].copy_(torch.as_tensor(logits32))
    layer.forward(dev(inp["x"]))
    assert api.read_device_status(layer.ws) == 0
    r = {k: v.cpu().numpy() for k, v in layer.routing.items()}
    S = int(ref["seg_off"][-1])
    assert 0 < S < T * K                                   # some pairs dropped
    for k in ("counts", "kept", "seg_off"):
        assert (r[k] == ref[k]).all(), k
    assert (r["slot_of"].reshape(T, K) == ref["slot_of"]).all()
    assert (r["perm"][:S] == ref["perm"]).all()
    st = layer.stats.cpu().numpy()
    assert (st[:E] == ref["f"].astype(np.float32)).all()
    assert np.max(np.abs(st[E:2 * E] - ref["P"])) <= 1e-6
    assert abs(st[2 * E] - ref["loss"]) <= 1e-6 * max(1.0, ref["loss"])
    _check_extended(st, E, logits32.astype(np.float64), ref["counts"], ref["kept"])


# ------------------------------------------------------------- expert FFNs
@pytest.mark.parametrize("name", list(SMALL))
def test_routed_expert_ffn_matches_oracle(name):
    cfg = SMALL[name]
    inp = inputs(name)
    ref = oracle_routing(cfg, given_logits(cfg).astype(np.float64), inp["sel_bias"])
    S = int(ref["seg_off"][-1])
    if S == 0:
        pytest.skip("everything dropped")
    prob = problem(cfg)
    ws = api.alloc_workspace(prob)
    R = api.max_rows(prob)
    x = inp["x"]
    tok = ref["perm"].astype(np.int64) // cfg.top_k
    x_rows = torch.zeros((R, cfg.d_model), dtype=x.dtype)
    x_rows[:S] = x[torch.as_tensor(tok)]
    y_rows = torch.zeros((R, cfg.d_model), dtype=x.dtype, device="cuda")
    api.reset_device_status(ws)
    api.moe_expert_ffn(prob, api.FFN_ROUTED, dev(x_rows), R, dev(ref["seg_off"]), dev(inp["w13"]), dev(inp["w2"]),
                       y_rows, ws)
    assert api.read_device_status(ws) == 0
    got = y_rows[:S].float().cpu().numpy()
    # oracle: each kept row through its expert, weight 1
    e_of = np.repeat(np.arange(cfg.n_experts), ref["kept"])
    w13, w2 = host_np(inp["w13"]), host_np(inp["w2"])
    xs = host_np(x)
    rows = sample_rows(S, 64, seed=1)
    want = np.stack([oracle.swiglu(_row64(xs, tok[r], x.dtype), w13[e_of[r]], w2[e_of[r]]) for r in rows])
    assert rel_err(got[rows], want) <= tol(cfg)


# last-tile row counts: every swap-tile MMA width class and token-box height,
# and groups of 256 h + r rows with small r (16, 17, 32, 33, 48, 49, 1)
REMAINDER_SIZES = [1, 15, 16, 17, 31, 33, 100, 128, 129, 200, 255, 256, 257, 300, 513, 0, 48,
                   272, 273, 288, 289, 304, 305, 560, 561]


def _remainder_ffn(F, sizes=REMAINDER_SIZES):
    E, d = len(sizes), 256
    T = sum(sizes)
    prob = api.make_problem(T, d, E, 1, F, 0, 0.0, "bf16")
    ws = api.alloc_workspace(prob)
    R = api.max_rows(prob)
    g = torch.Generator().manual_seed(21)
    x_rows = torch.randn((R, d), generator=g).to(torch.bfloat16)
    w13 = (torch.randn((E, 2 * F, d), generator=g) / d ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn((E, d, F), generator=g) / F ** 0.5).to(torch.bfloat16)
    seg_off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    y_rows = torch.zeros((R, d), dtype=torch.bfloat16, device="cuda")
    api.reset_device_status(ws)
    api.moe_expert_ffn(prob, api.FFN_ROUTED, dev(x_rows), R, dev(seg_off), dev(w13), dev(w2), y_rows, ws)
    assert api.read_device_status(ws) == 0
    return y_rows[:T].cpu(), (x_rows, w13, w2, seg_off)


@pytest.mark.parametrize("F", [200, 320])
@pytest.mark.parametrize("tile,swap", [("256all", ""), ("256all", "0"), ("256all", "100"), ("128", "")])
def test_routed_ffn_every_remainder_shape(tile, swap, F, monkeypatch):
    """Groups whose last 256-row tile holds 1..256 rows (every swap-tile MMA
    width class and token-box height, ragged F across two column tiles), after
    zero to two full tiles, every row against the oracle's SwiGLU of its
    expert.  F = 320 (a multiple of 64) takes the down projection's
    chunk-merged swap-tile boxes, F = 200 the per-chunk ones (the up
    projection, d = 256, always merged)."""
    monkeypatch.setenv("MOE_B200_GEMM_TILE", tile)
    monkeypatch.setenv("MOE_B200_SWAP_MAX", swap)
    y, (x_rows, w13, w2, seg_off) = _remainder_ffn(F)
    sizes = REMAINDER_SIZES
    E, T = len(sizes), sum(sizes)
    got = y.float().numpy()
    xs, a, b = host_np(x_rows), host_np(w13), host_np(w2)
    e_of = np.repeat(np.arange(E), sizes)
    want = np.stack([oracle.swiglu(_row64(xs, r, torch.bfloat16), a[e_of[r]], b[e_of[r]]) for r in range(T)])
    assert rel_err(got, want) <= 2e-2
    for e in range(E):   # per group too, so a small group is not hidden by a large one
        lo, hi = seg_off[e], seg_off[e + 1]
        if hi > lo:
            assert rel_err(got[lo:hi], want[lo:hi]) <= 2e-2, (e, sizes[e])


def _row64(xs, t, dtype):
    if dtype == torch.bfloat16:
        return (xs[t].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return xs[t].astype(np.float64)


@pytest.mark.parametrize("name", [n for n, c in SMALL.items() if c.n_shared > 0])
def test_shared_expert_ffn_matches_oracle(name):
    cfg = SMALL[name]
    inp = inputs(name)
    prob = problem(cfg)
    ws = api.alloc_workspace(prob)
    y = torch.zeros((cfg.T, cfg.d_model), dtype=inp["x"].dtype, device="cuda")
    api.moe_expert_ffn(prob, api.FFN_SHARED, dev(inp["x"]), cfg.T, None, dev(inp["w13_shared"]),
                       dev(inp["w2_shared"]), y, ws)
    got = y.float().cpu().numpy()
    xs = host_np(inp["x"])
    a, b = host_np(inp["w13_shared"]), host_np(inp["w2_shared"])
    rows = sample_rows(cfg.T, 64, seed=2)
    want = np.stack([sum(oracle.swiglu(_row64(xs, t, inp["x"].dtype), a[s], b[s]) for s in range(cfg.n_shared))
                     for t in rows])
    assert rel_err(got[rows], want) <= tol(cfg)


# ------------------------------------------------------------------ combine
@pytest.mark.parametrize("name", ["mini_mixtral", "mini_zen", "ragged_f32", "ragged_bf16", "tiny_capacity"])
def test_combine_matches_oracle(name):
    cfg = SMALL[name]
    inp = inputs(name)
    ref = oracle_routing(cfg, given_logits(cfg).astype(np.float64), inp["sel_bias"])
    prob = problem(cfg)
    ws = api.alloc_workspace(prob)
    R = max(api.max_rows(prob), 1)
    gen = torch.Generator().manual_seed(5)
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    y_perm = torch.randn((R, cfg.d_model), generator=gen).to(tdt)
    y_sh = torch.randn((cfg.T, cfg.d_model), generator=gen).to(tdt) if cfg.n_shared else None
    w32 = ref["w"].astype(np.float32)
    y = torch.empty((cfg.T, cfg.d_model), dtype=tdt, device="cuda")
    api.moe_combine(prob, dev(y_perm), dev(ref["slot_of"]), dev(w32), dev(y_sh), y, ws)
    want = oracle.combine(host_np(y_perm), ref["slot_of"], w32.astype(np.float64),
                          None if y_sh is None else host_np(y_sh))
    got = y.float().cpu().numpy()
    # one rounding of an fp32 sum: half an ulp of the output type, plus fp32 accumulation
    ulp = 2.0 ** -8 if cfg.dtype == "bf16" else 2.0 ** -23
    assert np.all(np.abs(got - want) <= ulp * np.abs(want) + 1e-6 * np.max(np.abs(want)))


# ------------------------------------------------------------- whole layer
@pytest.mark.parametrize("name", list(SMALL))
def test_layer_forward_given_logits_matches_oracle(name):
    cfg = SMALL[name]
    inp = inputs(name)
    logits32 = given_logits(cfg)
    ref = oracle_routing(cfg, logits32.astype(np.float64), inp["sel_bias"])
    layer = MoeLayer.from_inputs(inp, flags=api.FLAG_LOGITS_GIVEN)
    layer.routing["logits"].copy_(torch.as_tensor(logits32))
    y = layer.forward(dev(inp["x"]))
    assert api.read_device_status(layer.ws) == 0
    r = {k: v.cpu().numpy() for k, v in layer.routing.items()}
    assert (r["topk_idx"] == ref["idx"]).all()
    assert (r["counts"] == ref["counts"]).all() and (r["kept"] == ref["kept"]).all()
    assert (r["seg_off"] == ref["seg_off"]).all() and (r["slot_of"] == ref["slot_of"]).all()
    S = int(ref["seg_off"][-1])
    assert (r["perm"][:S] == ref["perm"]).all()
    want = oracle_layer(inp, ref)
    assert rel_err(y.float().cpu().numpy(), want) <= tol(cfg)
    # dropped pairs contribute nothing: tokens with every pair dropped and no
    # shared expert come out exactly zero
    all_dropped = (ref["slot_of"] < 0).all(1)
    if cfg.n_shared == 0 and all_dropped.any():
        assert (y[torch.as_tensor(all_dropped).cuda()] == 0).all()


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_forward_end_to_end_matches_oracle(name):
    """GPU computes its own logits.  Routing must agree with the oracle's own
    float64 routing except at near-ties (score gap within the logit error);
    outputs agree on every token whose routing agrees."""
    cfg = SMALL[name]
    inp = inputs(name)
    layer = MoeLayer.from_inputs(inp)
    y = layer.forward(dev(inp["x"]))
    assert api.read_device_status(layer.ws) == 0
    l64 = oracle.gate_logits(host_np(inp["x"]), host_np(inp["w_gate"]), inp["logit_offset"])
    ref = oracle_routing(cfg, l64, inp["sel_bias"])
    g_idx = layer.routing["topk_idx"].cpu().numpy()
    g_slot = layer.routing["slot_of"].cpu().numpy()
    same = (g_idx == ref["idx"]).all(1) & ((g_slot >= 0) == (ref["slot_of"] >= 0)).all(1)
    assert same.mean() >= 0.97, f"routing agreed on {same.mean():.4f} of tokens"
    want = oracle_layer(inp, ref)
    got = y.float().cpu().numpy()
    assert rel_err(got[same], want[same]) <= tol(cfg)


def test_layer_forward_is_deterministic():
    cfg = SMALL["mini_skewed"]
    inp = inputs("mini_skewed")
    layer = MoeLayer.from_inputs(inp)
    x = dev(inp["x"])
    y1 = layer.forward(x).clone()
    s1 = layer.stats.clone()
    r1 = {k: v.clone() for k, v in layer.routing.items()}
    y2 = layer.forward(x)
    assert torch.equal(y1, y2) and torch.equal(s1, layer.stats)
    for k, v in layer.routing.items():
        assert torch.equal(r1[k], v), k


@pytest.mark.parametrize("name", ["mini_mixtral", "mini_zen", "mini_decode", "ragged_bf16"])
def test_clocked_forward_equals_the_plain_forward_and_stamps_its_stages(name):
    """moe_layer_forward_clocked runs the same kernels (plus two atomics per
    CTA): outputs, routing and statistics bit-identical to moe_layer_forward,
    and every BF16 stage that ran has a span, in order along the stream."""
    from sparse_mixture_experts_04_b200 import _lib
    inp = inputs(name)
    layer = MoeLayer.from_inputs(inp)
    x = dev(inp["x"])
    y1 = layer.forward(x).clone()
    s1 = layer.stats.clone()
    r1 = {k: v.clone() for k, v in layer.routing.items()}
    clocks = torch.zeros(2 * _lib.NUM_CLOCKS, dtype=torch.int64, device="cuda")
    y2 = torch.empty_like(y1)
    api.moe_layer_forward_clocked(layer.prob, x, layer.weights, y2, layer.routing, layer.stats, layer.ws, clocks)
    torch.cuda.synchronize()
    assert api.read_device_status(layer.ws) == 0
    assert torch.equal(y1, y2) and torch.equal(s1, layer.stats)
    for k, v in layer.routing.items():
        assert torch.equal(r1[k], v), k
    us = api.stage_clock_us(clocks.cpu().tolist())
    for st in ("route", "dispatch", "gather", "up", "down", "combine"):
        assert us[st] is not None and 0.0 < us[st] < 1e5, (st, us)
    c = [int(v) & 0xFFFFFFFFFFFFFFFF for v in clocks.cpu().tolist()]
    names = _lib.CLOCK_NAMES
    start = lambda n: (~c[2 * names.index(n)]) & 0xFFFFFFFFFFFFFFFF
    end = lambda n: c[2 * names.index(n) + 1]
    # each stage starts reading only after its predecessor's last CTA ended
    order = ["route", "dispatch", "gather", "up", "down", "combine"]
    for a, b in zip(order, order[1:]):
        assert end(a) <= start(b), (a, b)


def test_layer_stats_match_oracle_and_uniform_routing_gives_alpha():
    # all-equal logits: P_e = 1/E for every expert; with K = E every expert is
    # chosen by every token, so f_e = 1/E too, and the loss is exactly alpha
    cfg = MoeConfig("uniform", T=96, d_model=64, n_experts=8, top_k=8, d_ff=64, n_shared=0, capacity_factor=0.0,
                    dtype="bf16", seed=3)
    idx, w, stats = _route_given(cfg, np.zeros((96, 8), np.float32), None)
    assert np.allclose(stats[:8], 1 / 8, atol=0) and np.allclose(stats[8:16], 1 / 8, atol=1e-7)
    assert abs(stats[16] - 0.01) <= 1e-8


# --------------------------------------------------- both GEMM tile shapes
@pytest.mark.parametrize("tile,swap", [("128", ""), ("256", ""), ("256all", "0"), ("256all", "64"), ("256all", "")])
@pytest.mark.parametrize("name", ["mini_mixtral", "mini_zen", "ragged_bf16", "mini_skewed", "mini_decode"])
def test_layer_forward_both_tile_shapes(name, tile, swap, monkeypatch):
    """The 128-row single-CTA and 256-row CTA-pair expert GEMMs, each forced,
    the pair kernel with and without operand-swapped remainder tiles, against
    the oracle (the library picks one per problem size otherwise)."""
    monkeypatch.setenv("MOE_B200_GEMM_TILE", tile)
    monkeypatch.setenv("MOE_B200_SWAP_MAX", swap)
    cfg = SMALL[name]
    inp = inputs(name)
    logits32 = given_logits(cfg)
    ref = oracle_routing(cfg, logits32.astype(np.float64), inp["sel_bias"])
    layer = MoeLayer.from_inputs(inp, flags=api.FLAG_LOGITS_GIVEN)
    layer.routing["logits"].copy_(torch.as_tensor(logits32))
    y = layer.forward(dev(inp["x"]))
    assert api.read_device_status(layer.ws) == 0
    assert rel_err(y.float().cpu().numpy(), oracle_layer(inp, ref)) <= tol(cfg)


@pytest.mark.parametrize("tile", ["256all", "128"])
@pytest.mark.parametrize("name", ["mini_zen", "ragged_bf16", "mini_decode"])
def test_mixed_shared_launch_is_bit_identical_to_separate_launches(name, tile, monkeypatch):
    """With one tile shape forced for both FFNs (CTA pairs, or single CTAs)
    the shared experts run in the routed experts' launches, their tiles
    interleaved with the routed ones; each tile is computed as in separate
    launches, so the layer output and the statistics are the same bytes.
    Also against the oracle."""
    monkeypatch.setenv("MOE_B200_GEMM_TILE", tile)
    cfg = SMALL[name]
    inp = inputs(name)
    logits32 = given_logits(cfg)
    outs = []
    for mix in ("1", "0"):
        monkeypatch.setenv("MOE_B200_MIX_SHARED", mix)
        layer = MoeLayer.from_inputs(inp, flags=api.FLAG_LOGITS_GIVEN)
        layer.routing["logits"].copy_(torch.as_tensor(logits32))
        y = layer.forward(dev(inp["x"]))
        assert api.read_device_status(layer.ws) == 0
        outs.append((y.clone(), layer.stats.clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    ref = oracle_routing(cfg, logits32.astype(np.float64), inp["sel_bias"])
    assert rel_err(outs[0][0].float().cpu().numpy(), oracle_layer(inp, ref)) <= tol(cfg)


@pytest.mark.parametrize("name", ["mini_mixtral", "mini_zen", "mini_skewed", "mini_decode", "ragged_bf16"])
def test_deep_swap_stages_are_bit_identical(name, monkeypatch):
    """Swap tiles of at most 64 token rows take 192-deep stages (three 64-deep
    chunks per stage slot); the MMAs run in the same k order, so the layer
    output is the same bytes as with 128-deep stages (MOE_B200_DEEP_SWAP=0),
    with pair tiles forced and every remainder of up to 128 rows swapped."""
    monkeypatch.setenv("MOE_B200_GEMM_TILE", "256all")
    cfg = SMALL[name]
    inp = inputs(name)
    logits32 = given_logits(cfg)
    outs = []
    for deep in ("1", "0"):
        monkeypatch.setenv("MOE_B200_DEEP_SWAP", deep)
        layer = MoeLayer.from_inputs(inp, flags=api.FLAG_LOGITS_GIVEN)
        layer.routing["logits"].copy_(torch.as_tensor(logits32))
        y = layer.forward(dev(inp["x"]))
        assert api.read_device_status(layer.ws) == 0
        outs.append(y.clone())
    assert torch.equal(outs[0], outs[1])
    ref = oracle_routing(cfg, logits32.astype(np.float64), inp["sel_bias"])
    assert rel_err(outs[0].float().cpu().numpy(), oracle_layer(inp, ref)) <= tol(cfg)


def test_forward_host_pipelined_matches_device_forward():
    """MoeLayer.forward_host (host batches in and out, copies overlapped with
    the kernels on side streams) gives the same bytes as forward() per batch."""
    cfg = SMALL["mini_zen"]
    inp = inputs("mini_zen")
    layer = MoeLayer.from_inputs(inp)
    gen = torch.Generator().manual_seed(3)
    xs = [(torch.randn((cfg.T, cfg.d_model), generator=gen)).to(torch.bfloat16).pin_memory() for _ in range(5)]
    ys = [torch.empty((cfg.T, cfg.d_model), dtype=torch.bfloat16).pin_memory() for _ in range(5)]
    st = [torch.empty(2 * cfg.n_experts + 1, dtype=torch.float32).pin_memory() for _ in range(5)]
    layer.forward_host(xs, ys, st)
    for i in range(5):
        y = layer.forward(xs[i].cuda())
        assert torch.equal(ys[i], y.cpu()), i
        assert torch.equal(st[i], layer.stats.cpu()), i


# ------------------------------------------------- extended statistics (f1)
def _check_extended(stats, E, logits64, counts, kept):
    x = stats[2 * E + 1:]
    z = oracle.router_zloss(logits64)
    u = oracle.utilization(counts, kept)
    assert abs(x[0] - z) <= 1e-5 * max(1.0, abs(z))
    assert abs(x[1] - u["entropy_bits"]) <= 1e-5 * max(1.0, u["entropy_bits"])
    assert abs(x[2] - u["cv"]) <= 1e-5 * max(1.0, u["cv"])
    assert abs(x[3] - u["drop_rate"]) <= 1e-6
    assert x[4] == u["n_below_half"] and x[5] == u["n_above_double"]


@pytest.mark.parametrize("name", ["mini_mixtral", "mini_zen", "mini_skewed", "tiny_capacity", "wide_e256"])
def test_route_extended_stats_match_oracle(name):
    cfg = SMALL[name]
    inp = inputs(name)
    logits32 = given_logits(cfg)
    flags = api.FLAG_LOGITS_GIVEN | api.FLAG_EXTENDED_STATS
    ref = oracle_routing(cfg, logits32.astype(np.float64), inp["sel_bias"])
    prob = problem(cfg, flags)
    ws = api.alloc_workspace(prob)
    T, E, K = cfg.T, cfg.n_experts, cfg.top_k
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    stats = torch.empty(api.stats_size(prob), dtype=torch.float32, device="cuda")
    api.moe_route(prob, None, None, None, dev(inp["sel_bias"]), dev(logits32), idx, w, stats, ws)
    st = stats.cpu().numpy()
    assert (st[:E] == ref["f"].astype(np.float32)).all()
    _check_extended(st, E, logits32.astype(np.float64), ref["counts"], ref["kept"])


@pytest.mark.parametrize("name", ["mini_mixtral", "mini_zen", "ragged_f32", "tiny_capacity"])
def test_layer_extended_stats_match_oracle(name):
    cfg = SMALL[name]
    inp = inputs(name)
    logits32 = given_logits(cfg)
    ref = oracle_routing(cfg, logits32.astype(np.float64), inp["sel_bias"])
    layer = MoeLayer.from_inputs(inp, flags=api.FLAG_LOGITS_GIVEN | api.FLAG_EXTENDED_STATS)
    layer.routing["logits"].copy_(torch.as_tensor(logits32))
    layer.forward(dev(inp["x"]))
    st = layer.stats.cpu().numpy()
    E = cfg.n_experts
    assert st.shape[0] == 2 * E + 7
    assert np.max(np.abs(st[E:2 * E] - ref["P"])) <= 1e-6
    assert abs(st[2 * E] - ref["loss"]) <= 1e-6 * max(1.0, ref["loss"])
    _check_extended(st, E, logits32.astype(np.float64), ref["counts"], ref["kept"])
