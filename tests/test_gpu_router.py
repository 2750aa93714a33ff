"""The BF16 router with its own logits (tensor-core gate GEMM, then the
selection kernel) against the float64 oracle.

Bit-exact routing is checked on seeded inputs whose logits are exact in
float32 (small multiples of 1/8: every summation order, split-K included,
gives the same value, and ties are frequent), so the oracle computes the very
same logits."""
import numpy as np
import pytest
import torch

import oracle
from helpers import dev, host_np
from sparse_mixture_experts_04_b200 import api
from sparse_mixture_experts_04_b200.synth import exact_router_inputs

pytestmark = pytest.mark.gpu

CASES = [  # T, d, E, K, bias ("none" | "prob" | "logit"), offset
    (777, 256, 8, 2, "none", False),
    (300, 512, 16, 1, "none", True),
    (1000, 256, 60, 4, "prob", True),
    (513, 192, 128, 8, "prob", False),
    (257, 128, 128, 6, "logit", True),
    (200, 128, 256, 6, "prob", True),
    (129, 64, 256, 8, "none", False),
    (32, 4096, 128, 8, "prob", False),
    (1, 64, 4, 4, "none", True),
    (64, 1024, 64, 8, "logit", False),
    (100, 128, 256, 32, "prob", False),   # the largest top-K: K + 1 rounds exceed a warp's lanes
    (65, 64, 64, 32, "none", True),
]


def _route(prob, inp, sel_bias, T, E, K, extended):
    ws = api.alloc_workspace(prob)
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    stats = torch.empty(api.stats_size(prob), dtype=torch.float32, device="cuda")
    api.reset_device_status(ws)
    api.moe_route(prob, dev(inp["x"]), dev(inp["w_gate"]), dev(inp["logit_offset"]), dev(sel_bias), logits, idx, w,
                  stats, ws)
    assert api.read_device_status(ws) == 0
    return logits.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy(), stats.cpu().numpy()


@pytest.mark.parametrize("case", CASES, ids=[f"T{c[0]}-d{c[1]}-E{c[2]}-K{c[3]}-{c[4]}" for c in CASES])
def test_router_is_bit_exact_on_exact_logits(case):
    T, d, E, K, bias, with_off = case
    inp = exact_router_inputs(T, d, E, seed=T + E)
    if not with_off:
        inp["logit_offset"] = None
    rng = np.random.default_rng(E * 7 + K)
    sel_bias = None if bias == "none" else rng.uniform(-0.02, 0.02, size=E).astype(np.float32)
    flags = api.FLAG_EXTENDED_STATS | (api.FLAG_BIAS_LOGIT if bias == "logit" else 0)
    prob = api.make_problem(T, d, E, K, 64, 0, 1.0, "bf16", flags)
    logits, idx, w, stats = _route(prob, inp, sel_bias, T, E, K, True)
    l64 = oracle.gate_logits(host_np(inp["x"]), host_np(inp["w_gate"]), inp["logit_offset"])
    assert (logits.astype(np.float64) == l64).all()          # the logits are exact on both sides
    mode = oracle.BIAS_LOGIT if bias == "logit" else oracle.BIAS_PROB
    r_idx, r_w, p = oracle.select(l64, K, bias=sel_bias, bias_mode=mode)
    assert (idx == r_idx).all()
    assert np.max(np.abs(w - r_w)) <= 1e-6
    counts = np.bincount(r_idx.ravel(), minlength=E).astype(np.int32)
    f, P, loss = oracle.balance(counts, p, K, 0.01)
    assert (stats[:E] == f.astype(np.float32)).all()
    assert np.max(np.abs(stats[E:2 * E] - P)) <= 1e-6
    assert abs(stats[2 * E] - loss) <= 1e-6 * max(1.0, loss)
    z = oracle.router_zloss(l64)
    assert abs(stats[2 * E + 1] - z) <= 1e-5 * max(1.0, z)
