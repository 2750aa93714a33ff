"""The five workloads at full size, in the launch configuration the benchmark
times (one moe_layer_forward per step through MoeLayer).

Routing outputs are compared bit-exactly over every token (both sides fed the
same float32 logits); layer outputs on sampled tokens the oracle computes one
by one; the GPU's own gate logits on sampled tokens; and the GPU's end-to-end
routing against the oracle's own float64 routing."""
import gc

import numpy as np
import pytest
import torch

import oracle
from helpers import dev, generate, given_logits, host_np, oracle_layer, oracle_routing, rel_err, sample_rows, tol
from sparse_mixture_experts_04_b200 import MoeLayer, api
from sparse_mixture_experts_04_b200.synth import CONFIGS

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

N_SAMPLE = {"tiny_fp32": 64, "mixtral": 6, "zen_fine": 16, "skewed": 24, "decode": 32}


def slot_rows(ref: dict, K: int, per_tail: int = 4) -> tuple:
    """Tokens chosen by expert row (slot) rather than by token: for every
    expert, the owners of its first row, of the first row of its last full
    256-row tile, and of `per_tail` rows spread over its last row tile (all of
    them when it has fewer).  The last tile of at most 128 rows is the one the
    CTA-pair GEMM computes operand-swapped, so every expert's remainder tile is
    compared with the oracle at its real row count."""
    seg, perm = ref["seg_off"], ref["perm"]
    toks = set()
    for e in range(len(seg) - 1):
        lo, hi = int(seg[e]), int(seg[e + 1])
        n = hi - lo
        if n == 0:
            continue
        full = n // 256
        tail0 = lo + full * 256 if n % 256 else lo + max(full - 1, 0) * 256
        picks = {lo, lo + max(full - 1, 0) * 256}
        tail = np.arange(tail0, hi)
        picks |= set(int(r) for r in (tail if len(tail) <= per_tail else
                                      tail[np.linspace(0, len(tail) - 1, per_tail).astype(int)]))
        toks |= {int(perm[r]) // K for r in picks}
    return tuple(sorted(toks))


@pytest.fixture(scope="module", params=list(CONFIGS))
def workload(request):
    name = request.param
    cfg = CONFIGS[name]
    inp = generate(cfg)
    yield name, cfg, inp
    del inp
    gc.collect()
    torch.cuda.empty_cache()


def test_full_size_given_logits(workload):
    name, cfg, inp = workload
    logits32 = given_logits(cfg)
    ref = oracle_routing(cfg, logits32.astype(np.float64), inp["sel_bias"])
    layer = MoeLayer.from_inputs(inp, flags=api.FLAG_LOGITS_GIVEN | api.FLAG_EXTENDED_STATS)
    layer.routing["logits"].copy_(torch.as_tensor(logits32))
    y = layer.forward(dev(inp["x"]))
    assert api.read_device_status(layer.ws) == 0
    r = {k: v.cpu().numpy() for k, v in layer.routing.items()}
    assert (r["topk_idx"] == ref["idx"]).all()
    assert np.max(np.abs(r["topk_w"] - ref["w"])) <= 1e-6
    for k in ("counts", "kept", "seg_off", "slot_of"):
        assert (r[k] == ref[k]).all(), k
    S = int(ref["seg_off"][-1])
    assert (r["perm"][:S] == ref["perm"]).all()
    st = layer.stats.cpu().numpy()
    E = cfg.n_experts
    assert (st[:E] == ref["f"].astype(np.float32)).all()
    assert np.max(np.abs(st[E:2 * E] - ref["P"])) <= 1e-6
    assert abs(st[2 * E] - ref["loss"]) <= 1e-6 * max(1.0, ref["loss"])
    z = oracle.router_zloss(logits32.astype(np.float64))
    u = oracle.utilization(ref["counts"], ref["kept"])
    x = st[2 * E + 1:]
    assert abs(x[0] - z) <= 1e-5 * max(1.0, z)
    assert abs(x[1] - u["entropy_bits"]) <= 1e-5 * max(1.0, u["entropy_bits"])
    assert abs(x[2] - u["cv"]) <= 1e-5 * max(1.0, u["cv"]) and abs(x[3] - u["drop_rate"]) <= 1e-6
    assert x[4] == u["n_below_half"] and x[5] == u["n_above_double"]
    # sampled outputs, including tokens with dropped pairs when there are any
    dropped = np.nonzero((ref["slot_of"] < 0).any(1))[0][:4]
    by_slot = slot_rows(ref, cfg.top_k) if cfg.dtype == "bf16" else ()
    rows = sample_rows(cfg.T, N_SAMPLE[name], seed=cfg.seed, extra=tuple(int(t) for t in dropped) + by_slot)
    want = oracle_layer(inp, ref, rows=rows)
    got = y.float().cpu().numpy()[rows]
    assert rel_err(got, want) <= tol(cfg)


def test_full_size_end_to_end(workload):
    name, cfg, inp = workload
    layer = MoeLayer.from_inputs(inp)
    y = layer.forward(dev(inp["x"]))
    assert api.read_device_status(layer.ws) == 0
    g_logits = layer.routing["logits"].cpu().numpy().astype(np.float64)
    l64 = oracle.gate_logits(host_np(inp["x"]), host_np(inp["w_gate"]), inp["logit_offset"])
    bound = (1e-5 if cfg.dtype == "f32" else 1e-3) * max(1.0, float(np.max(np.abs(l64))))
    assert np.max(np.abs(g_logits - l64)) <= bound
    ref = oracle_routing(cfg, l64, inp["sel_bias"])
    g_idx = layer.routing["topk_idx"].cpu().numpy()
    g_slot = layer.routing["slot_of"].cpu().numpy()
    same = (g_idx == ref["idx"]).all(1) & ((g_slot >= 0) == (ref["slot_of"] >= 0)).all(1)
    assert same.mean() >= 0.99, f"routing agreed on {same.mean():.4f} of tokens"
    rows = sample_rows(cfg.T, N_SAMPLE[name], seed=cfg.seed + 100)
    rows = rows[same[rows]]
    want = oracle_layer(inp, ref, rows=rows)
    got = y.float().cpu().numpy()[rows]
    assert rel_err(got, want) <= tol(cfg)


def test_full_size_mixed_shared_launch_is_bit_identical(workload, monkeypatch):
    """Where the shared experts run in the routed experts' launches (zen_fine:
    both on CTA-pair tiles), every tile is computed as in separate launches:
    outputs and statistics are bit-identical with the mixing turned off."""
    name, cfg, inp = workload
    if cfg.dtype != "bf16" or cfg.n_shared == 0:
        pytest.skip("no shared experts on the tensor-core path")
    x = dev(inp["x"])
    outs = []
    for mix in ("1", "0"):
        monkeypatch.setenv("MOE_B200_MIX_SHARED", mix)
        layer = MoeLayer.from_inputs(inp)
        y = layer.forward(x)
        assert api.read_device_status(layer.ws) == 0
        outs.append((y.clone(), layer.stats.clone()))
        del layer
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
