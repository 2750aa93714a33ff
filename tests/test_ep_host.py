"""Expert-parallel forward, host side (no GPU): the exchange plan of the C
library (moe_ep_plan, a host function) and the schedule of
sparse_mixture_experts_04_b200.ep, run with the oracle as every rank's
compute -- in one process (ep.forward_emulated) and as gloo ranks
(ep.forward with torch.distributed point-to-point exchanges).

The reference is the single-device layer on each rank's batch ("Scaling with
experts", What you still pay for: the tokens travel to their experts' devices
and back, which changes where an expert runs, not what it computes), built
from the same oracle pieces, so the outputs must agree exactly."""
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_04_b200 import api, ep
from sparse_mixture_experts_04_b200.synth import MoeConfig, extra_activations, generate

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CFG = MoeConfig("ep_tiny", T=24, d_model=16, n_experts=8, top_k=2, d_ff=24, n_shared=1, capacity_factor=1.0,
                dtype="f32", seed=11, x_std=1.0)


# ---------------------------------------------------------------- the plan
def _random_seg_off(rng, G, E, T, K):
    out = np.zeros((G, E + 1), np.int32)
    for s in range(G):
        kept = rng.integers(0, T + 1, size=E)
        kept[rng.random(E) < 0.25] = 0            # empty experts
        kept = np.minimum(kept, T * K // E + 3)
        out[s, 1:] = np.cumsum(kept)
    return out


@pytest.mark.parametrize("G,E", [(1, 4), (2, 4), (2, 8), (4, 8), (8, 8), (3, 6)])
def test_plan_tables_match_their_definition(G, E):
    """One chunk per peer each way: the block of x_perm holding peer q's
    experts goes to q; the blocks received lie end to end in source order, and
    segment s*E_l + el covers source s's rows for local expert el."""
    rng = np.random.default_rng(G * 100 + E)
    so = _random_seg_off(rng, G, E, T=20, K=2)
    El = E // G
    for rank in range(G):
        send, recv, local = (t.numpy() for t in api.moe_ep_plan(G, rank, E, torch.from_numpy(so)))
        assert send.shape == (G, 3) and recv.shape == (G, 3) and local.shape == (G * El + 1,)
        for q in range(G):
            assert tuple(send[q]) == (q, so[rank, q * El], so[rank, (q + 1) * El] - so[rank, q * El])
        off = 0
        for s in range(G):
            rows = so[s, (rank + 1) * El] - so[s, rank * El]
            assert tuple(recv[s]) == (s, off, rows)
            for el in range(El):
                assert local[s * El + el] == off + so[s, rank * El + el] - so[s, rank * El]
            off += rows
        assert local[G * El] == off
        assert (np.diff(local) >= 0).all()


@pytest.mark.parametrize("G,E", [(2, 4), (4, 8), (3, 6), (8, 8)])
def test_plan_moves_every_kept_row_to_its_expert_and_back(G, E):
    """Simulate the exchange with labelled rows: each row of rank s's x_perm is
    (s, slot).  After the forward exchange, segment s*E_l + el of rank q's
    local buffer holds exactly the rows rank s kept for q's local expert el;
    after the return exchange every y_perm slot holds its own label again."""
    rng = np.random.default_rng(7 * G + E)
    so = _random_seg_off(rng, G, E, T=16, K=2)
    El = E // G
    plans = [tuple(t.numpy() for t in api.moe_ep_plan(G, r, E, torch.from_numpy(so))) for r in range(G)]
    x_perm = [np.array([(s, i) for i in range(so[s, E])], dtype=np.int64).reshape(-1, 2) for s in range(G)]
    x_loc = [np.full((plans[q][2][-1], 2), -1, np.int64) for q in range(G)]
    for s in range(G):          # forward: one message s -> q
        for q in range(G):
            out = [(o, n) for p, o, n in plans[s][0] if p == q and n > 0]
            inn = [(o, n) for p, o, n in plans[q][1] if p == s and n > 0]
            assert [n for _, n in out] == [n for _, n in inn] and len(out) <= 1
            for (o1, n), (o2, _) in zip(out, inn):
                x_loc[q][o2:o2 + n] = x_perm[s][o1:o1 + n]
    for q in range(G):
        local = plans[q][2]
        for s in range(G):
            for el in range(El):
                e = q * El + el
                want = [(s, i) for i in range(so[s, e], so[s, e + 1])]
                seg = s * El + el
                assert [tuple(r) for r in x_loc[q][local[seg]:local[seg + 1]]] == want
    y_perm = [np.full((so[s, E], 2), -1, np.int64) for s in range(G)]
    for q in range(G):          # back: the expert outputs (here: the labels) return to their sources
        for s in range(G):
            out = [(o, n) for p, o, n in plans[q][1] if p == s and n > 0]
            inn = [(o, n) for p, o, n in plans[s][0] if p == q and n > 0]
            for (o1, n), (o2, _) in zip(out, inn):
                y_perm[s][o2:o2 + n] = x_loc[q][o1:o1 + n]
    for s in range(G):
        assert np.array_equal(y_perm[s], x_perm[s])


def test_plan_rejects_bad_arguments():
    so = torch.zeros((2, 5), dtype=torch.int32)
    with pytest.raises(api.MoeError):
        api.moe_ep_plan(2, 2, 4, so)            # rank out of range
    with pytest.raises(api.MoeError):
        api.moe_ep_plan(3, 0, 4, torch.zeros((3, 5), dtype=torch.int32))   # E % G != 0
    bad = torch.tensor([[0, 2, 1, 3, 4], [0, 0, 0, 0, 0]], dtype=torch.int32)
    with pytest.raises(api.MoeError):
        api.moe_ep_plan(2, 0, 4, bad)           # decreasing offsets
    bad = torch.tensor([[1, 2, 3, 3, 4], [0, 0, 0, 0, 0]], dtype=torch.int32)
    with pytest.raises(api.MoeError):
        api.moe_ep_plan(2, 1, 4, bad)           # not starting at 0
    L = api._lib.lib()
    assert L.moe_ep_plan(1, 0, 4, None, None, None, None) == -1


# ------------------------------------------------- the schedule with oracle compute
class OracleExperts:
    """One rank's compute written with the oracle (float64), with the buffer
    names of ep.CudaExperts; test infrastructure only."""

    def __init__(self, cfg, inp, n_ranks, rank):
        T, E, K, d, F = cfg.T, cfg.n_experts, cfg.top_k, cfg.d_model, cfg.d_ff
        self.cfg, self.inp = cfg, inp
        self.prob = api.make_problem(T, d, E, K, F, cfg.n_shared, cfg.capacity_factor, cfg.dtype)
        self.n_ranks, self.rank, self.n_local = n_ranks, rank, E // n_ranks
        self.d_model, self.dtype, self.device = d, torch.float64, torch.device("cpu")
        self.cap = oracle.capacity(T, K, E, cfg.capacity_factor)
        f64 = dict(dtype=torch.float64)
        self.x_perm, self.y_perm = torch.zeros((T * K, d), **f64), torch.zeros((T * K, d), **f64)
        self.x_loc = torch.zeros((n_ranks * T * K, d), **f64)
        self.y_loc = torch.zeros((n_ranks * T * K, d), **f64)
        lo = rank * self.n_local
        self.w13 = inp["w13"][lo:lo + self.n_local].numpy()
        self.w2 = inp["w2"][lo:lo + self.n_local].numpy()

    def route_dispatch(self, x):
        logits = oracle.gate_logits(x.numpy(), self.inp["w_gate"].numpy())
        self.idx, self.w, _ = oracle.select(logits, self.cfg.top_k)
        self.disp = oracle.dispatch(self.idx, self.cfg.n_experts, self.cap)
        perm = self.disp["perm"]
        self.x_perm[:len(perm)] = torch.from_numpy(x.numpy().astype(np.float64)[perm // self.cfg.top_k])
        return torch.from_numpy(self.disp["seg_off"])

    def experts(self, n_rows, local_seg_off):
        lso = local_seg_off.tolist()
        for seg in range(len(lso) - 1):      # segment i: local expert i % E_l
            el = seg % self.n_local
            for r in range(lso[seg], lso[seg + 1]):
                self.y_loc[r] = torch.from_numpy(oracle.swiglu(self.x_loc[r].numpy(), self.w13[el], self.w2[el]))

    def shared(self, x):
        self.ysh = None
        if self.cfg.n_shared:
            xs = x.numpy().astype(np.float64)
            self.ysh = np.stack([sum(oracle.swiglu(xs[t], self.inp["w13_shared"][s].numpy(),
                                                   self.inp["w2_shared"][s].numpy())
                                     for s in range(self.cfg.n_shared)) for t in range(self.cfg.T)])

    def combine(self, y):
        n = int(self.disp["seg_off"][-1])
        y.copy_(torch.from_numpy(oracle.combine(self.y_perm[:max(n, 1)].numpy(), self.disp["slot_of"], self.w,
                                                self.ysh)))


def single_device_reference(cfg, inp, x):
    """The same oracle pieces with every expert on one device."""
    one = OracleExperts(cfg, inp, 1, 0)
    rk = ep.EpRank(one)
    return ep.forward_emulated([rk], [x])[0], one


def _inputs(cfg, G):
    inp = generate(cfg)
    xs = extra_activations(cfg, G)
    return inp, xs


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_emulated_ranks_equal_the_single_device_layer(G):
    inp, xs = _inputs(CFG, G)
    ranks = [ep.EpRank(OracleExperts(CFG, inp, G, r)) for r in range(G)]
    ys = ep.forward_emulated(ranks, xs)
    for r in range(G):
        want, one = single_device_reference(CFG, inp, xs[r])
        assert torch.equal(ys[r], want)
        # and the oracle's own whole-layer definition
        ref = oracle.layer_rows(xs[r].numpy(), inp["w13"].numpy(), inp["w2"].numpy(), one.idx, one.w,
                                one.disp["slot_of"], w13_shared=inp["w13_shared"].numpy(),
                                w2_shared=inp["w2_shared"].numpy())
        assert np.max(np.abs(ys[r].numpy() - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))
    # some pairs were dropped by the capacity and every rank received rows
    assert any(int(rk.k.disp["counts"].sum()) > int(rk.k.disp["seg_off"][-1]) for rk in ranks)
    assert all(int(rk.local_seg_off[-1]) > 0 for rk in ranks)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        inp, xs = _inputs(CFG, world)
        rk = ep.EpRank(OracleExperts(CFG, inp, world, rank))
        y = ep.forward(rk, xs[rank])
        want, _ = single_device_reference(CFG, inp, xs[rank])
        q.put((rank, bool(torch.equal(y, want)), int(rk.local_seg_off[-1])))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_equal_the_single_device_layer(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[0] for o in out] == list(range(world))
    assert all(o[1] for o in out), out
    assert all(o[2] > 0 for o in out)


# ------------------------------------------- the peer-memory form: buffer tables across processes
class _FakeIpc:
    """Stands in for api.IpcBuffer on CPU: an allocation gets an address that
    encodes (owner rank, buffer kind) and a handle that carries it; mapping a
    handle gives the owner's address back, as CUDA IPC maps the same memory."""
    rank = 0
    made = []
    release_order = []

    def __init__(self, shape, dtype, handle=None):
        if handle is None:
            kind = sum(1 for b in _FakeIpc.made if not b.opened)
            self.ptr = 1_000_000 * (_FakeIpc.rank + 1) + kind
            self.opened = False
        else:
            self.ptr = int.from_bytes(handle[:8], "little")
            self.opened = True
        self.tensor = torch.zeros(shape, dtype=dtype)
        self.released = False
        _FakeIpc.made.append(self)

    def handle(self):
        return self.ptr.to_bytes(8, "little") + bytes(api.IPC_HANDLE_BYTES - 8)

    def release(self):
        self.released = True
        _FakeIpc.release_order.append(self)


class _Kernels:
    def __init__(self, world, rank):
        self.n_ranks, self.rank, self.prob = world, rank, api.make_problem(8, 16, 2 * world, 1, 16)
        self.n_local, self.max_local_rows, self.d_model = 2, 5, 16
        self.dtype, self.device = torch.float32, torch.device("cpu")
        self.x_loc = self.y_loc = None


def _peer_table_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        _FakeIpc.rank = rank
        api.IpcBuffer = _FakeIpc          # this process only (spawned)
        rk = ep.PeerRank(_Kernels(world, rank))
        ep.open_peer_buffers(rk)
        own = [b.ptr for b in _FakeIpc.made if not b.opened]
        q.put((rank, rk.recv_ptrs.tolist(), rk.out_ptrs.tolist(), own,
               tuple(rk.k.x_loc.shape), len(rk.ipc)))
        rk.release()
        assert all(b.released for b in _FakeIpc.made)
        # the peers' mappings were closed before this rank's own buffers were freed
        order = [b.opened for b in _FakeIpc.release_order]
        assert order == sorted(order, reverse=True)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_open_peer_buffers_tables_list_every_rank_in_order(world):
    """ep.open_peer_buffers on gloo ranks with a stand-in for the IPC calls:
    every rank's receive and output tables hold, at index q, rank q's own
    buffers (its own allocations at its own index, the peers' mapped from
    their handles), and each rank keeps 2 + 2 (G - 1) mappings to release."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_peer_table_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    owners = {r: own for r, _, _, own, _, _ in out}
    for r, recv, outp, own, shape, n_ipc in out:
        assert recv == [owners[s][0] for s in range(world)]
        assert outp == [owners[s][1] for s in range(world)]
        assert shape == (5, 16) and n_ipc == 2 * world
