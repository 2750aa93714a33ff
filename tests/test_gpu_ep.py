"""Expert-parallel forward on the GPU: G ranks' expert sets, each with its own
batch, run through the expert-parallel schedule (ep.forward_emulated: the
ranks live in one process and every exchange is a device copy; with one GPU
no two processes may wait on each other), and a one-rank NCCL process group
through ep.forward.  Each rank's output is checked against the oracle's
layer on that rank's batch and against the single-device library layer
(MoeLayer with all E experts).  All compute runs in libmoe_b200.so."""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch

from helpers import dev, generate, oracle_layer, rel_err, tol
from sparse_mixture_experts_04_b200 import MoeLayer, api, ep
from sparse_mixture_experts_04_b200.synth import MoeConfig, extra_activations

pytestmark = pytest.mark.gpu

CFGS = {
    # several tiles per expert and a ragged tail; capacity drops some pairs
    "small": MoeConfig("ep_small", T=320, d_model=256, n_experts=8, top_k=2, d_ff=384, n_shared=1,
                       capacity_factor=1.0, dtype="bf16", seed=21, x_std=1.0),
    # groups of a few hundred rows (pair tiles), no capacity limit, no shared expert
    "pairs": MoeConfig("ep_pairs", T=1536, d_model=512, n_experts=8, top_k=2, d_ff=1024, n_shared=0,
                       capacity_factor=0.0, dtype="bf16", seed=22, x_std=1.0),
}


def _reference(inp, x, k):
    """Oracle layer on this batch for the routing the rank computed (the
    routing itself is compared with the single-device layer's)."""
    route = dict(idx=k.topk_idx.cpu().numpy(), w=k.topk_w.cpu().numpy().astype(np.float64),
                 slot_of=k.slot_of.cpu().numpy())
    return oracle_layer(dict(inp, x=x), route)


def _single_device(cfg, inp, x):
    layer = MoeLayer.from_inputs(inp)
    y = layer.forward(dev(x))
    torch.cuda.synchronize()
    return y, layer


def _ranks(cfg, inp, G):
    P = api.make_problem(cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff, cfg.n_shared,
                         cfg.capacity_factor, cfg.dtype, 0, cfg.alpha)
    full = {k: dev(inp[k]) for k in ("w_gate", "w13", "w2", "w13_shared", "w2_shared")}
    return [ep.EpRank(ep.CudaExperts(P, ep.split_weights(full, G, r), G, r)) for r in range(G)]


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("name", list(CFGS))
def test_emulated_ranks_match_oracle_and_single_device(name, G):
    cfg = CFGS[name]
    inp = generate(cfg)
    xs = extra_activations(cfg, G)
    ranks = _ranks(cfg, inp, G)
    ys = ep.forward_emulated(ranks, [dev(x) for x in xs])
    torch.cuda.synchronize()
    for r in range(G):
        k = ranks[r].k
        assert api.read_device_status(k.ws) == 0 and api.read_device_status(k.ws_local) == 0
        y_one, layer = _single_device(cfg, inp, xs[r])
        # same routing as the single-device layer on this batch
        for key in ("topk_idx", "seg_off", "slot_of"):
            assert torch.equal(getattr(k, key), layer.routing[key]), key
        want = _reference(inp, xs[r], k)
        got = ys[r].float().cpu().numpy()
        assert rel_err(got, want) <= tol(cfg), (r, rel_err(got, want))
        # the expert rows are grouped differently (sources side by side), so a
        # row may sit in another tile shape than on one device: BF16-level agreement
        assert rel_err(got, y_one.float().cpu().numpy()) <= 1e-2
        assert int(ranks[r].local_seg_off[-1]) > 0
    # every kept row went out and came back exactly once
    total_kept = sum(int(rk.k.seg_off[-1]) for rk in ranks)
    assert sum(int(rk.local_seg_off[-1]) for rk in ranks) == total_kept


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_group_matches_single_device():
    import torch.distributed as dist
    cfg = CFGS["small"]
    inp = generate(cfg)
    x = extra_activations(cfg, 1)[0]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        rk = _ranks(cfg, inp, 1)[0]
        y = ep.forward(rk, dev(x))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    y_one, _ = _single_device(cfg, inp, x)
    want = _reference(inp, x, rk.k)
    got = y.float().cpu().numpy()
    assert rel_err(got, want) <= tol(cfg)
    # one rank: the local rows are x_perm itself, in the same order and tiles
    assert torch.equal(y, y_one)


@pytest.mark.parametrize("tile", ["256all", "128"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_expert_ffn_segments_repeat_the_experts(dtype, tile, monkeypatch):
    """moe_expert_ffn_segments: segment i of the rows uses expert i % E (the
    expert-parallel receive buffer: one block per source, experts in order
    inside it), checked row by row against the oracle, empty segments and
    segments of several hundred rows included."""
    import oracle
    from helpers import host_np
    if tile:
        monkeypatch.setenv("MOE_B200_GEMM_TILE", tile)
    E, S, d, F = 4, 12, 256, 192
    rng = np.random.default_rng(31)
    rows = rng.integers(0, 120, size=S)
    rows[[2, 7]] = 0
    rows[5] = 300
    seg = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    n = int(seg[-1])
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = torch.from_numpy(rng.normal(size=(n, d)).astype(np.float32)).to(tdt)
    w13 = torch.from_numpy((rng.normal(size=(E, 2 * F, d)) / np.sqrt(d)).astype(np.float32)).to(tdt)
    w2 = torch.from_numpy((rng.normal(size=(E, d, F)) / np.sqrt(F)).astype(np.float32)).to(tdt)
    prob = api.make_problem(n, d, E, 1, F, 0, 0.0, dtype)
    ws = api.alloc_workspace(prob)
    y = torch.zeros((n, d), dtype=tdt, device="cuda")
    api.reset_device_status(ws)
    api.moe_expert_ffn_segments(prob, dev(x), n, dev(seg), S, dev(w13), dev(w2), y, ws)
    assert api.read_device_status(ws) == 0
    xs, a, b = host_np(x), host_np(w13), host_np(w2)
    if dtype == "bf16":
        x64 = (xs.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    else:
        x64 = xs.astype(np.float64)
    e_of = np.repeat(np.arange(S) % E, rows)
    pick = np.unique(np.concatenate([seg[:-1][rows > 0], seg[1:][rows > 0] - 1, rng.choice(n, 48, replace=False)]))
    want = np.stack([oracle.swiglu(x64[r], a[e_of[r]], b[e_of[r]]) for r in pick])
    got = y.float().cpu().numpy()[pick]
    assert rel_err(got, want) <= (2e-2 if dtype == "bf16" else 1e-4)
