"""GPU parity of the load-balancing steps between forwards: per-expert
capacities in the dispatch (Zen MoDE §5.3 capacity_e), the selection-bias
update (Zen-Max §2.3) and the adaptive capacity (Zen MoDE §5.3 C_e), against
the float64 oracle.  Integer results bit-exact; the float32 biases bit-exact
(both sides round the same float64 expression once)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import dev, generate, given_logits, host_np, oracle_layer, problem, rel_err, sample_rows, tol
from sparse_mixture_experts_04_b200 import MoeLayer, api
from sparse_mixture_experts_04_b200.synth import MoeConfig

pytestmark = pytest.mark.gpu

CFGS = {
    "mixtral_like": MoeConfig("mixtral_like", T=1031, d_model=256, n_experts=8, top_k=2, d_ff=384, n_shared=0,
                              capacity_factor=1.0, dtype="bf16", seed=41),
    "zen_like": MoeConfig("zen_like", T=700, d_model=256, n_experts=128, top_k=8, d_ff=128, n_shared=2,
                          capacity_factor=1.0, dtype="bf16", seed=42, bias_range=0.1),
    "skew_e64": MoeConfig("skew_e64", T=2000, d_model=128, n_experts=64, top_k=4, d_ff=136, n_shared=0,
                          capacity_factor=1.0, dtype="bf16", seed=43, zipf_s=1.2),
    "e256": MoeConfig("e256", T=300, d_model=128, n_experts=256, top_k=6, d_ff=64, n_shared=0,
                      capacity_factor=2.0, dtype="bf16", seed=44, bias_range=0.01),
}


def _caps(E, T, seed):
    """Seeded per-expert capacities: no limit (-1), zero, small, large, and above T."""
    rng = np.random.default_rng(seed)
    caps = rng.integers(0, max(4, 3 * T // E), size=E).astype(np.int32)
    caps[rng.choice(E, size=max(1, E // 8), replace=False)] = -1
    caps[rng.choice(E, size=max(1, E // 16), replace=False)] = 0
    caps[0] = T + 5
    return caps


@pytest.mark.parametrize("name", list(CFGS))
def test_dispatch_capacity_is_bit_exact(name):
    cfg = CFGS[name]
    inp = generate(cfg)
    T, E, K = cfg.T, cfg.n_experts, cfg.top_k
    idx, _, _ = oracle.select(given_logits(cfg).astype(np.float64), K)
    caps = _caps(E, T, cfg.seed)
    want = oracle.dispatch_caps(idx, E, caps.astype(np.int64))
    prob = problem(cfg, api.FLAG_EXPERT_CAPACITY)
    ws = api.alloc_workspace(prob)
    i32 = dict(dtype=torch.int32, device="cuda")
    counts, kept = torch.empty(E, **i32), torch.empty(E, **i32)
    seg_off, slot_of = torch.empty(E + 1, **i32), torch.empty((T, K), **i32)
    perm = torch.full((api.max_rows(prob),), -7, **i32)
    x = dev(inp["x"])
    x_perm = torch.empty((api.max_rows(prob), cfg.d_model), dtype=x.dtype, device="cuda")
    api.reset_device_status(ws)
    api.moe_dispatch_capacity(prob, dev(idx), dev(caps), x, counts, kept, seg_off, slot_of, perm, x_perm, ws)
    assert api.read_device_status(ws) == 0
    for k, v in (("counts", counts), ("kept", kept), ("seg_off", seg_off), ("slot_of", slot_of)):
        assert (v.cpu().numpy() == want[k]).all(), k
    S = int(want["seg_off"][-1])
    assert (perm.cpu().numpy()[:S] == want["perm"]).all()
    assert (perm.cpu().numpy()[S:] == -7).all()
    rows = want["perm"] // K
    assert torch.equal(x_perm[:S].cpu(), torch.as_tensor(inp["x"])[torch.as_tensor(rows)])


@pytest.mark.parametrize("name", list(CFGS))
@pytest.mark.parametrize("mode", [api.BIAS_UPDATE_SIGN, api.BIAS_UPDATE_PROPORTIONAL])
def test_bias_update_is_bit_exact(name, mode):
    cfg = CFGS[name]
    T, E, K = cfg.T, cfg.n_experts, cfg.top_k
    rng = np.random.default_rng(cfg.seed + mode)
    prob = problem(cfg)
    bias = rng.normal(scale=0.05, size=E).astype(np.float32)
    b_dev = dev(bias)
    want = bias.copy()
    for step in range(5):
        counts = rng.multinomial(T * K, rng.dirichlet(np.ones(E))).astype(np.int32)
        if step == 2 and (T * K) % E == 0:
            counts[:] = (T * K) // E          # every expert on target: no change
        api.moe_balance_update(prob, dev(counts), b_dev, 3e-3, mode)
        want = oracle.bias_update(counts, T * K, want, 3e-3, mode)
        got = b_dev.cpu().numpy()
        assert (got.view(np.uint32) == want.view(np.uint32)).all(), f"step {step}"


@pytest.mark.parametrize("name", list(CFGS))
@pytest.mark.parametrize("window", [1, 3])
def test_adaptive_capacity_is_bit_exact_over_a_rolling_window(name, window):
    cfg = CFGS[name]
    T, E, K = cfg.T, cfg.n_experts, cfg.top_k
    rng = np.random.default_rng(cfg.seed + 10 * window)
    prob = problem(cfg)
    hist = torch.zeros((window, E), dtype=torch.int32, device="cuda")
    caps = torch.empty(E, dtype=torch.int32, device="cuda")
    seen = []
    for step in range(7):
        counts = rng.multinomial(T * K, rng.dirichlet(np.full(E, 0.5))).astype(np.int32)
        seen.append(counts)
        gamma = [0.0, 2.0, 8.0, -1.5][step % 4]
        api.moe_balance_update(prob, dev(counts), None, 0.0, 0, hist, step, 1.25, gamma, caps)
        want = oracle.adaptive_capacity(T, K, np.stack(seen[-window:]), 1.25, gamma)
        assert (caps.cpu().numpy() == want).all(), f"step {step}"


@pytest.mark.parametrize("name", ["mixtral_like", "zen_like"])
def test_layer_with_per_expert_capacity(name):
    """A whole forward with per-expert capacities: routing bit-exact (given
    logits), the statistics' drop figures, and outputs on sampled tokens."""
    cfg = CFGS[name]
    inp = generate(cfg)
    T, E, K = cfg.T, cfg.n_experts, cfg.top_k
    logits32 = given_logits(cfg)
    caps = _caps(E, T, cfg.seed + 1)
    layer = MoeLayer.from_inputs(inp, flags=api.FLAG_LOGITS_GIVEN | api.FLAG_EXPERT_CAPACITY | api.FLAG_EXTENDED_STATS)
    layer.weights["expert_capacity"].copy_(torch.as_tensor(caps))
    layer.routing["logits"].copy_(torch.as_tensor(logits32))
    y = layer.forward(dev(inp["x"]))
    assert api.read_device_status(layer.ws) == 0
    bm = oracle.BIAS_PROB
    idx, w, p = oracle.select(logits32.astype(np.float64), K, bias=inp["sel_bias"], bias_mode=bm)
    disp = oracle.dispatch_caps(idx, E, caps.astype(np.int64))
    r = {k: v.cpu().numpy() for k, v in layer.routing.items()}
    assert (r["topk_idx"] == idx).all()
    for k in ("counts", "kept", "seg_off", "slot_of"):
        assert (r[k] == disp[k]).all(), k
    u = oracle.utilization(disp["counts"], disp["kept"])
    st = layer.stats.cpu().numpy()[2 * E + 1:]
    assert abs(st[3] - u["drop_rate"]) <= 1e-6
    route = dict(idx=idx, w=w, slot_of=disp["slot_of"])
    rows = sample_rows(T, 24, seed=cfg.seed, extra=tuple(np.nonzero((disp["slot_of"] < 0).any(1))[0][:4]))
    want = oracle_layer(inp, route, rows=rows)
    assert rel_err(y.float().cpu().numpy()[rows], want) <= tol(cfg)


def test_layer_balance_loop_matches_oracle():
    """Several forwards with MoeLayer.balance_update between them: bias and
    capacities follow the oracle's closed loop step for step."""
    cfg = CFGS["skew_e64"]
    inp = generate(cfg)
    T, E, K = cfg.T, cfg.n_experts, cfg.top_k
    sel_bias = np.zeros(E, np.float32)
    inp = dict(inp, sel_bias=sel_bias)
    layer = MoeLayer.from_inputs(inp, flags=api.FLAG_LOGITS_GIVEN | api.FLAG_EXPERT_CAPACITY)
    logits32 = given_logits(cfg)
    layer.routing["logits"].copy_(torch.as_tensor(logits32))
    b = sel_bias.copy()
    cap_now = np.full(E, oracle.capacity(T, K, E, cfg.capacity_factor), np.int64)
    seen = []
    x = dev(inp["x"])
    for step in range(6):
        layer.forward(x)
        idx, _, _ = oracle.select(logits32.astype(np.float64), K, bias=b, bias_mode=oracle.BIAS_PROB)
        disp = oracle.dispatch_caps(idx, E, cap_now)
        assert (layer.routing["topk_idx"].cpu().numpy() == idx).all(), f"step {step}"
        assert (layer.routing["kept"].cpu().numpy() == disp["kept"]).all(), f"step {step}"
        layer.balance_update(bias_rate=0.01, bias_mode=api.BIAS_UPDATE_SIGN, gamma=4.0, window=2)
        b = oracle.bias_update(disp["counts"], T * K, b, 0.01, oracle.BIAS_UPDATE_SIGN)
        seen.append(disp["counts"])
        cap_now = oracle.adaptive_capacity(T, K, np.stack(seen[-2:]), cfg.capacity_factor, 4.0)
        assert (layer.weights["sel_bias"].cpu().numpy() == b).all()
        assert (layer.weights["expert_capacity"].cpu().numpy() == cap_now).all()
    assert api.read_device_status(layer.ws) == 0
