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
    # FP32 (CUDA-core expert GEMMs), ragged d and F
    "f32": MoeConfig("ep_f32", T=200, d_model=72, n_experts=8, top_k=2, d_ff=40, n_shared=1,
                     capacity_factor=1.0, dtype="f32", seed=23, x_std=0.5),
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


# ------------------------------------------------------------ the exchange over peer memory
def _plan_reference(seg_all, rank):
    """The receive layout written out: expert-major receive buffers, source
    ranks in order within an expert; returns (delta [E], local_seg_off)."""
    G, E1 = seg_all.shape
    E, El = E1 - 1, (E1 - 1) // G
    rows = seg_all[:, 1:].astype(np.int64) - seg_all[:, :-1]          # [G, E]
    tot = rows.sum(axis=0)
    delta = np.zeros(E, np.int64)
    for e in range(E):
        q = e // El
        base = tot[q * El:e].sum()
        delta[e] = base + rows[:rank, e].sum() - seg_all[rank, e]
    own = tot[rank * El:(rank + 1) * El]
    local = np.concatenate([[0], np.cumsum(own)]).astype(np.int32)
    return delta, local


@pytest.mark.parametrize("G,E", [(1, 8), (2, 8), (4, 64), (8, 256), (8, 8)])
def test_peer_plan_matches_its_definition(G, E):
    rng = np.random.default_rng(G * 1000 + E)
    counts = rng.integers(0, 40, size=(G, E))
    counts[:, rng.integers(0, E)] = 0                                   # an expert nobody chose
    seg_all = np.concatenate([np.zeros((G, 1), np.int64), np.cumsum(counts, axis=1)], axis=1).astype(np.int32)
    sa = torch.as_tensor(seg_all).cuda()
    for rank in range(G):
        delta = torch.empty(E, dtype=torch.int64, device="cuda")
        local = torch.empty(E // G + 1, dtype=torch.int32, device="cuda")
        api.moe_ep_peer_plan(G, rank, E, sa, delta, local)
        want_d, want_l = _plan_reference(seg_all, rank)
        assert (delta.cpu().numpy() == want_d).all()
        assert (local.cpu().numpy() == want_l).all()
    # every slot of every rank lands on a distinct row of its owner's buffer
    El = E // G
    for q in range(G):
        seen = []
        for r in range(G):
            d_r, _ = _plan_reference(seg_all, r)
            for e in range(q * El, (q + 1) * El):
                seen += [j + d_r[e] for j in range(seg_all[r, e], seg_all[r, e + 1])]
        assert sorted(seen) == list(range(int(counts[:, q * El:(q + 1) * El].sum())))


def _peer_ranks(cfg, inp, G):
    ranks = [ep.PeerRank(rk.k) for rk in _ranks(cfg, inp, G)]
    ep.connect_emulated(ranks)
    return ranks


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("name", list(CFGS))
def test_emulated_peer_exchange_equals_the_copy_schedule(name, G):
    """Scatter into the experts' ranks' buffers, local experts over the
    expert-major buffer, combine from the owners' outputs: the rows reach the
    expert GEMM in the order the copy schedule's regrouping gives them, and the
    combine adds the same terms in the same order, so every rank's output is
    the same bytes as ep.forward_emulated's; and within the layer's tolerance
    of the oracle."""
    cfg = CFGS[name]
    inp = generate(cfg)
    xs = [dev(x) for x in extra_activations(cfg, G)]
    ys_copy = [y.clone() for y in ep.forward_emulated(_ranks(cfg, inp, G), xs)]
    ranks = _peer_ranks(cfg, inp, G)
    ys = ep.forward_emulated_p2p(ranks, xs)
    torch.cuda.synchronize()
    for r in range(G):
        k = ranks[r].k
        assert api.read_device_status(k.ws) == 0 and api.read_device_status(k.ws_local) == 0
        assert torch.equal(ys[r], ys_copy[r]), r
        want = _reference(inp, xs[r].cpu(), k)
        assert rel_err(ys[r].float().cpu().numpy(), want) <= tol(cfg)
    # the receive buffers hold every kept row once
    assert sum(int(rk.local_seg_off[-1]) for rk in ranks) == sum(int(rk.k.seg_off[-1]) for rk in ranks)
    # a second forward on the same buffers gives the same outputs
    ys2 = ep.forward_emulated_p2p(ranks, xs)
    for r in range(G):
        assert torch.equal(ys2[r], ys[r])


def test_one_rank_nccl_group_peer_exchange():
    """forward_p2p through a one-rank NCCL group: IPC-allocated receive and
    output buffers, the all-gather into device memory, the device plan and
    the two stream barriers; equal to the copy schedule's ep.forward."""
    import torch.distributed as dist
    cfg = CFGS["small"]
    inp = generate(cfg)
    x = dev(extra_activations(cfg, 1)[0])
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    rk = None
    try:
        y_copy = ep.forward(_ranks(cfg, inp, 1)[0], x).clone()
        rk = ep.PeerRank(_ranks(cfg, inp, 1)[0].k)
        ep.open_peer_buffers(rk)
        y = ep.forward_p2p(rk, x).clone()
        y2 = ep.forward_p2p(rk, x).clone()
        torch.cuda.synchronize()
    finally:
        if rk is not None:
            rk.release()
        dist.destroy_process_group()
    assert torch.equal(y, y_copy) and torch.equal(y2, y)
    assert rel_err(y.float().cpu().numpy(), _reference(inp, x.cpu(), rk.k)) <= tol(cfg)


def test_scatter_into_a_buffer_mapped_from_another_process():
    """CUDA IPC on one GPU: this process allocates a receive buffer
    (moe_ipc_malloc) and hands its handle to a second process, which maps it
    (moe_ipc_open) and runs moe_ep_scatter into it; the rows arrive here."""
    import subprocess
    import sys
    n, d, seed = 300, 264, 5
    buf = api.IpcBuffer((n, d), torch.bfloat16)
    try:
        buf.tensor.zero_()
        torch.cuda.synchronize()
        child = os.path.join(os.path.dirname(os.path.abspath(__file__)), "ep_ipc_child.py")
        r = subprocess.run([sys.executable, child, buf.handle().hex(), str(n), str(d), str(seed)],
                           capture_output=True, text=True, timeout=300)
        assert r.returncode == 0, r.stderr[-2000:]
        g = torch.Generator().manual_seed(seed)
        want = torch.randn((n, d), generator=g).to(torch.bfloat16)
        assert torch.equal(buf.tensor.cpu(), want)
    finally:
        buf.release()


@pytest.mark.parametrize("G", [2, 8])
def test_emulated_peer_exchange_with_per_expert_capacity(G):
    """MOE_FLAG_EXPERT_CAPACITY (Zen MoDE §5.3, a capacity per expert, some 0):
    each rank ranks with moe_dispatch_capacity; the peer-memory schedule equals
    the copy schedule byte for byte and the oracle on the rows each rank kept."""
    cfg = CFGS["small"]
    inp = generate(cfg)
    xs = [dev(x) for x in extra_activations(cfg, G)]
    rng = np.random.default_rng(G)
    caps = rng.integers(0, 3 * cfg.T * cfg.top_k // cfg.n_experts, size=cfg.n_experts).astype(np.int32)
    caps[1] = 0

    def ranks(peer):
        P = api.make_problem(cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff, cfg.n_shared,
                             cfg.capacity_factor, cfg.dtype, api.FLAG_EXPERT_CAPACITY, cfg.alpha)
        full = {k: dev(inp[k]) for k in ("w_gate", "w13", "w2", "w13_shared", "w2_shared")}
        full["expert_capacity"] = torch.as_tensor(caps).cuda()
        ks = [ep.CudaExperts(P, ep.split_weights(full, G, r), G, r) for r in range(G)]
        if not peer:
            return [ep.EpRank(k) for k in ks]
        out = [ep.PeerRank(k) for k in ks]
        ep.connect_emulated(out)
        return out

    ys_copy = [y.clone() for y in ep.forward_emulated(ranks(False), xs)]
    rk = ranks(True)
    ys = ep.forward_emulated_p2p(rk, xs)
    torch.cuda.synchronize()
    for r in range(G):
        k = rk[r].k
        assert (k.kept.cpu().numpy() <= caps).all() and int(k.kept[1]) == 0
        assert torch.equal(ys[r], ys_copy[r]), r
        assert rel_err(ys[r].float().cpu().numpy(), _reference(inp, xs[r].cpu(), k)) <= tol(cfg)
