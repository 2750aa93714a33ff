"""Expert-parallel forward of the MoE layer: the experts are partitioned over
G devices and each token's rows travel to the device holding its expert and
back ("Scaling with experts", What you still pay for; Zen MoDE §7.2
Communication Overhead (Distributed Training): an all-to-all between the
expert devices).

Rank q holds the global experts [q*E_l, (q+1)*E_l), E_l = E/G, plus a copy
of the router and of the shared experts.  One forward on rank q:

  1. moe_route + moe_dispatch on its own T tokens with the full router, so the
     capacity cut and the statistics are exactly those of a single device on
     that batch; the kept rows of global expert e sit in x_perm at
     seg_off[e] .. seg_off[e+1];
  2. all-gather of the G segment-offset vectors (E+1 int32 each) and
     moe_ep_plan (host): which rows go where;
  3. exchange: the rows for peer q's experts are one contiguous block of
     x_perm (seg_off[q E_l] .. seg_off[(q+1) E_l]), sent as one message; the
     blocks received lie end to end in rank order (source-major);
  4. moe_expert_ffn_segments with the local E_l experts over the G E_l row
     segments of that buffer (segment s E_l + el: source s, local expert el);
  5. exchange back: each source's block of outputs returns as one message to
     its y_perm, in the place its input came from;
  6. shared experts (local; `forward` runs them while the rows of step 3 are
     in flight) and moe_combine, as on one device.

Every step of the layer runs in libmoe_b200.so; this module allocates
buffers, computes nothing and moves rows with torch.distributed point-to-point
operations (NCCL between GPUs, gloo between CPU processes), or with device
copies for the chunks a rank keeps for itself.  `forward_emulated` runs the
same schedule for G ranks held in one process (every exchange a copy).

The second schedule (`PeerRank`, `forward_p2p`, `forward_emulated_p2p`, at the
end of this module) moves the rows inside the kernels instead: the dispatch
writes them into the experts' ranks' memory and the combine reads the outputs
from there, with a device-side plan and no host round trip.
"""
from __future__ import annotations

import torch

from . import api


class CudaExperts:
    """One rank's device state and kernels (C ABI): router + dispatch over the
    global E experts, the rank's E_l local experts, shared experts, combine.

    weights: w_gate [E, d], optional logit_offset / sel_bias [E],
    expert_capacity [E] (with FLAG_EXPERT_CAPACITY), w13 [E_l, 2F, d],
    w2 [E_l, d, F] (this rank's experts: global expert rank*E_l + i is local
    expert i), optional w13_shared / w2_shared."""

    def __init__(self, prob: api.MoeProblem, weights: dict, n_ranks: int, rank: int, device="cuda"):
        E, T, K, d, F = prob.n_experts, prob.T, prob.top_k, prob.d_model, prob.d_ff
        if n_ranks < 1 or not 0 <= rank < n_ranks or E % n_ranks:
            raise ValueError(f"{E} experts cannot be split over {n_ranks} ranks (rank {rank})")
        if prob.flags & api.FLAG_SAVE_GU:
            raise ValueError("FLAG_SAVE_GU belongs to the training layer; the expert-parallel path is forward only")
        self.prob, self.weights = prob, weights
        self.n_ranks, self.rank = n_ranks, rank
        self.n_local = E // n_ranks
        self.device = torch.device(device)
        self.dtype = torch.bfloat16 if prob.dtype == api.DTYPE_BF16 else torch.float32
        self.d_model = d
        if tuple(weights["w13"].shape) != (self.n_local, 2 * F, d) or tuple(weights["w2"].shape) != (self.n_local, d, F):
            raise ValueError(f"rank {rank} needs w13 [{self.n_local}, {2 * F}, {d}] and w2 [{self.n_local}, {d}, {F}]")
        self.capacity_flag = bool(prob.flags & api.FLAG_EXPERT_CAPACITY)
        if self.capacity_flag and weights.get("expert_capacity") is None:
            raise ValueError("FLAG_EXPERT_CAPACITY needs weights['expert_capacity'] [E]")
        # rows one source can send here: at most T*K, at most T per expert, at most the capacity
        cap = api.capacity(prob)
        per_src = min(T * K, self.n_local * T)
        if cap >= 0 and not self.capacity_flag:
            per_src = min(per_src, self.n_local * cap)
        self.max_local_rows = max(n_ranks * per_src, 1)
        # the local experts' problem: max_local_rows rows over E_l groups (top_k 1, no capacity)
        self.prob_local = api.make_problem(self.max_local_rows, d, self.n_local, 1, F, 0, 0.0, prob.dtype, 0,
                                           prob.alpha)
        dev = self.device
        i32 = dict(dtype=torch.int32, device=dev)
        self.ws = api.alloc_workspace(prob, dev)
        self.ws_local = api.alloc_workspace(self.prob_local, dev)
        mr = max(api.max_rows(prob), 1)
        self.logits = torch.empty((T, E), dtype=torch.float32, device=dev)
        self.topk_idx = torch.empty((T, K), **i32)
        self.topk_w = torch.empty((T, K), dtype=torch.float32, device=dev)
        self.counts, self.kept = torch.empty(E, **i32), torch.empty(E, **i32)
        self.seg_off = torch.empty(E + 1, **i32)
        self.slot_of = torch.empty((T, K), **i32)
        self.perm = torch.empty(mr, **i32)
        self.x_perm = torch.empty((mr, d), dtype=self.dtype, device=dev)
        self.y_perm = torch.empty((mr, d), dtype=self.dtype, device=dev)
        self.x_loc = torch.empty((self.max_local_rows, d), dtype=self.dtype, device=dev)
        self.y_loc = torch.empty((self.max_local_rows, d), dtype=self.dtype, device=dev)
        self.stats = torch.empty(api.stats_size(prob), dtype=torch.float32, device=dev)
        # segment offsets of the receive buffer: host plan -> pinned staging -> device, without a host wait
        self.seg_host = torch.empty(n_ranks * self.n_local + 1, dtype=torch.int32,
                                    pin_memory=self.device.type == "cuda")
        self.seg_dev = torch.empty(n_ranks * self.n_local + 1, **i32)
        self.y_shared = torch.empty((T, d), dtype=self.dtype, device=dev) if prob.n_shared > 0 else None

    def route_dispatch(self, x: torch.Tensor) -> torch.Tensor:
        w, P = self.weights, self.prob
        api.moe_route(P, x, w.get("w_gate"), w.get("logit_offset"), w.get("sel_bias"), self.logits, self.topk_idx,
                      self.topk_w, self.stats, self.ws)
        if self.capacity_flag:
            api.moe_dispatch_capacity(P, self.topk_idx, w["expert_capacity"], x, self.counts, self.kept,
                                      self.seg_off, self.slot_of, self.perm, self.x_perm, self.ws)
        else:
            api.moe_dispatch(P, self.topk_idx, x, self.counts, self.kept, self.seg_off, self.slot_of, self.perm,
                             self.x_perm, self.ws)
        return self.seg_off

    def route_rank(self, x: torch.Tensor) -> torch.Tensor:
        """Routing and the dispatch's ranks only (no gather): the peer-memory
        exchange moves the rows itself; returns this rank's seg_off [E+1]."""
        w, P = self.weights, self.prob
        api.moe_route(P, x, w.get("w_gate"), w.get("logit_offset"), w.get("sel_bias"), self.logits, self.topk_idx,
                      self.topk_w, self.stats, self.ws)
        if self.capacity_flag:
            api.moe_dispatch_capacity(P, self.topk_idx, w["expert_capacity"], x, self.counts, self.kept,
                                      self.seg_off, self.slot_of, self.perm, None, self.ws)
        else:
            api.moe_dispatch(P, self.topk_idx, x, self.counts, self.kept, self.seg_off, self.slot_of, self.perm,
                             None, self.ws)
        return self.seg_off

    def experts(self, n_rows: int, local_seg_off: torch.Tensor) -> None:
        """The local experts over the receive buffer's G E_l source-major
        segments (segment i: local expert i % E_l).  The offsets reach the
        device by an asynchronous copy from pinned memory; the next plan is
        made only after the next step's all-gather has been read on the host,
        which orders it after this copy."""
        if n_rows > 0:
            self.seg_host.copy_(local_seg_off)
            self.seg_dev.copy_(self.seg_host, non_blocking=True)
            api.moe_expert_ffn_segments(self.prob_local, self.x_loc, n_rows, self.seg_dev, self.seg_dev.numel() - 1,
                                        self.weights["w13"], self.weights["w2"], self.y_loc, self.ws_local)

    def shared(self, x: torch.Tensor) -> None:
        """The shared experts on this rank's batch (no routed rows needed)."""
        w, P = self.weights, self.prob
        if self.y_shared is not None:
            api.moe_expert_ffn(P, api.FFN_SHARED, x, P.T, None, w["w13_shared"], w["w2_shared"], self.y_shared,
                               self.ws)

    def combine(self, y: torch.Tensor) -> None:
        P = self.prob
        api.moe_combine(P, self.y_perm, self.slot_of, self.topk_w, self.y_shared, y, self.ws)


class EpRank:
    """The expert-parallel schedule of one rank, in phases (route, plan,
    exchange lists, experts, combine) so that a process-group driver and the
    in-process emulation share it.  `kernels` holds the rank's buffers
    (x_perm, y_perm, x_loc, y_loc, seg_off) and its compute (CudaExperts)."""

    def __init__(self, kernels):
        self.k = kernels
        self.send = self.recv = self.local_seg_off = None

    def route(self, x: torch.Tensor) -> torch.Tensor:
        """Steps 1: routing and dispatch; returns this rank's seg_off [E+1]."""
        return self.k.route_dispatch(x)

    def plan(self, seg_off_all: torch.Tensor) -> None:
        """Step 2: seg_off_all [G, E+1] int32 (host) of every rank."""
        self.send, self.recv, self.local_seg_off = api.moe_ep_plan(self.k.n_ranks, self.k.rank,
                                                                   self.k.prob.n_experts, seg_off_all)
        n = int(self.local_seg_off[-1])
        if n > self.k.x_loc.shape[0]:
            raise RuntimeError(f"rank {self.k.rank} would receive {n} rows, more than its bound "
                               f"{self.k.x_loc.shape[0]}")

    def _chunks(self, table, buf):
        return [(int(p), buf[int(o): int(o) + int(r)]) for p, o, r in table.tolist() if r > 0]

    def forward_lists(self):
        """Step 3: (sends, recvs) as lists of (peer, rows view)."""
        return self._chunks(self.send, self.k.x_perm), self._chunks(self.recv, self.k.x_loc)

    def experts(self) -> None:
        """Step 4."""
        self.k.experts(int(self.local_seg_off[-1]), self.local_seg_off)

    def backward_lists(self):
        """Step 5: the outputs go back the way the inputs came."""
        return self._chunks(self.recv, self.k.y_loc), self._chunks(self.send, self.k.y_perm)

    def shared(self, x: torch.Tensor) -> None:
        """Step 6a: the shared experts (independent of the exchange, so a
        process-group forward runs them while the rows are in flight)."""
        self.k.shared(x)

    def combine(self, y: torch.Tensor | None = None) -> torch.Tensor:
        """Step 6b: the gate-weighted combine."""
        if y is None:
            y = torch.empty((self.k.prob.T, self.k.d_model), dtype=self.k.dtype, device=self.k.device)
        self.k.combine(y)
        return y

    def finish(self, x: torch.Tensor, y: torch.Tensor | None = None) -> torch.Tensor:
        """Step 6: shared experts and the gate-weighted combine."""
        self.shared(x)
        return self.combine(y)


def _exchange(sends, recvs, rank: int, group=None, wait: bool = True):
    """Point-to-point exchange of row chunks; chunks a rank sends to itself are
    copied locally.  Messages between two ranks match in posting order.  With
    wait=False the requests are returned for the caller to wait on."""
    import torch.distributed as dist

    def glob(r):
        return r if group is None else dist.get_global_rank(group, r)

    self_out = [t for p, t in sends if p == rank]
    self_in = [t for p, t in recvs if p == rank]
    if len(self_out) != len(self_in):
        raise RuntimeError(f"rank {rank}: {len(self_out)} chunks to itself but {len(self_in)} expected")
    for a, b in zip(self_out, self_in):
        if a.shape != b.shape:
            raise RuntimeError(f"rank {rank}: self chunk of {a.shape[0]} rows into a slot of {b.shape[0]}")
        b.copy_(a)
    ops = [dist.P2POp(dist.isend, t, glob(p), group) for p, t in sends if p != rank]
    ops += [dist.P2POp(dist.irecv, t, glob(p), group) for p, t in recvs if p != rank]
    reqs = dist.batch_isend_irecv(ops) if ops else []
    if wait:
        for req in reqs:
            req.wait()
        return []
    return reqs


def forward(rank_state: EpRank, x: torch.Tensor, y: torch.Tensor | None = None, group=None) -> torch.Tensor:
    """One expert-parallel forward on this process's rank (torch.distributed
    initialised; NCCL for CUDA tensors).  Every rank of the group calls it
    with its own batch x [T, d]; returns this rank's layer output [T, d]."""
    import torch.distributed as dist
    k = rank_state.k
    G = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if G != k.n_ranks or rank != k.rank:
        raise RuntimeError(f"process group rank {rank}/{G} but the experts were placed for {k.rank}/{k.n_ranks}")
    seg = rank_state.route(x)
    parts = [torch.empty_like(seg) for _ in range(G)]
    dist.all_gather(parts, seg, group=group)
    rank_state.plan(torch.stack(parts).cpu())
    reqs = _exchange(*rank_state.forward_lists(), rank, group, wait=False)
    rank_state.shared(x)  # overlaps the rows in flight
    for req in reqs:
        req.wait()
    rank_state.experts()
    _exchange(*rank_state.backward_lists(), rank, group)
    return rank_state.combine(y)


def _emulated_exchange(lists) -> None:
    G = len(lists)
    for s in range(G):
        for r in range(G):
            out = [t for p, t in lists[s][0] if p == r]
            inn = [t for p, t in lists[r][1] if p == s]
            if len(out) != len(inn):
                raise RuntimeError(f"{len(out)} chunks {s}->{r} but {len(inn)} expected")
            for a, b in zip(out, inn):
                if a.shape != b.shape:
                    raise RuntimeError(f"chunk {s}->{r} of {a.shape[0]} rows into a slot of {b.shape[0]}")
                b.copy_(a)


def forward_emulated(ranks: list, xs: list) -> list:
    """The schedule of `forward` for G ranks held in one process (for example
    G ranks' expert sets on one device): every exchange is a copy.  Returns
    the G layer outputs."""
    if len(ranks) != len(xs):
        raise ValueError("one batch per rank")
    segs = [rk.route(x) for rk, x in zip(ranks, xs)]
    host = torch.stack([s.cpu() for s in segs])
    for rk in ranks:
        rk.plan(host)
    _emulated_exchange([rk.forward_lists() for rk in ranks])
    for rk in ranks:
        rk.experts()
    _emulated_exchange([rk.backward_lists() for rk in ranks])
    return [rk.finish(x) for rk, x in zip(ranks, xs)]


def split_weights(weights: dict, n_ranks: int, rank: int) -> dict:
    """This rank's share of a full weight set: its E/G routed experts (views),
    the router and the shared experts whole."""
    E = weights["w13"].shape[0]
    if E % n_ranks:
        raise ValueError(f"{E} experts cannot be split over {n_ranks} ranks")
    El = E // n_ranks
    out = {k: v for k, v in weights.items() if k not in ("w13", "w2")}
    out["w13"] = weights["w13"][rank * El:(rank + 1) * El].contiguous()
    out["w2"] = weights["w2"][rank * El:(rank + 1) * El].contiguous()
    return out


# ------------------------------------------------------------------------------------------
# The exchange over peer memory: the dispatch writes each kept row straight into the
# receive buffer of its expert's rank (moe_ep_scatter), and the combine reads each
# expert output from the rank that computed it (moe_ep_combine) -- loads and stores to
# peer memory inside the kernels.  The receive buffer is expert-major (local expert el's
# rows from source 0, then source 1, ...), so the local experts run as one group each
# (moe_expert_ffn over E_l groups, no regrouping), and the plan is a device kernel
# (moe_ep_peer_plan) on the all-gathered segment offsets: no host round trip.


class PeerRank:
    """One rank of the peer-memory schedule.  `kernels` (CudaExperts) holds the
    rank's routing buffers and its receive / output buffers x_loc / y_loc;
    connect() gives it every rank's x_loc and y_loc addresses (rank q's
    buffers at index q: local tensors in one process, mapped peer memory
    across processes)."""

    def __init__(self, kernels: CudaExperts):
        k = self.k = kernels
        dev = k.device
        self.delta = torch.empty(k.prob.n_experts, dtype=torch.int64, device=dev)
        self.local_seg_off = torch.empty(k.n_local + 1, dtype=torch.int32, device=dev)
        self.recv_ptrs = self.out_ptrs = None
        self.ipc = []

    def connect(self, recv_ptrs, out_ptrs) -> None:
        G = self.k.n_ranks
        if len(recv_ptrs) != G or len(out_ptrs) != G:
            raise ValueError(f"{G} ranks need {G} receive and {G} output buffers")
        self.recv_ptrs = torch.tensor([int(p) for p in recv_ptrs], dtype=torch.int64, device=self.k.device)
        self.out_ptrs = torch.tensor([int(p) for p in out_ptrs], dtype=torch.int64, device=self.k.device)

    def route(self, x: torch.Tensor) -> torch.Tensor:
        return self.k.route_rank(x)

    def plan(self, seg_off_all: torch.Tensor) -> None:
        """seg_off_all [G, E+1] int32 on the device (every rank's seg_off)."""
        k = self.k
        api.moe_ep_peer_plan(k.n_ranks, k.rank, k.prob.n_experts, seg_off_all, self.delta, self.local_seg_off)

    def scatter(self, x: torch.Tensor) -> None:
        k = self.k
        api.moe_ep_scatter(k.prob, k.n_ranks, x, k.perm, k.seg_off, self.recv_ptrs, self.delta)

    def experts(self) -> None:
        k = self.k
        api.moe_expert_ffn(k.prob_local, api.FFN_ROUTED, k.x_loc, k.max_local_rows, self.local_seg_off,
                           k.weights["w13"], k.weights["w2"], k.y_loc, k.ws_local)

    def shared(self, x: torch.Tensor) -> None:
        self.k.shared(x)

    def combine(self, y: torch.Tensor | None = None) -> torch.Tensor:
        k = self.k
        if y is None:
            y = torch.empty((k.prob.T, k.d_model), dtype=k.dtype, device=k.device)
        api.moe_ep_combine(k.prob, k.n_ranks, self.out_ptrs, self.delta, k.topk_idx, k.slot_of, k.topk_w,
                           k.y_shared, y)
        return y

    def release(self, group=None) -> None:
        """Unmap the peers' buffers, wait until every rank has unmapped this
        rank's (a barrier of the process group, when one is initialised), then
        free this rank's own (open_peer_buffers).  Every rank calls it."""
        opened = [b for b in self.ipc if b.opened]
        own = [b for b in self.ipc if not b.opened]
        for b in opened:
            b.release()
        if own:
            import torch.distributed as dist
            if dist.is_available() and dist.is_initialized():
                dist.barrier(group=group)
        for b in own:
            b.release()
        self.ipc = []


def connect_emulated(ranks: list) -> None:
    """G PeerRanks held in one process: every rank's table points at the
    others' local buffers."""
    recv = [rk.k.x_loc.data_ptr() for rk in ranks]
    out = [rk.k.y_loc.data_ptr() for rk in ranks]
    for rk in ranks:
        rk.connect(recv, out)


def forward_emulated_p2p(ranks: list, xs: list) -> list:
    """The peer-memory schedule for G ranks held in one process (connect_emulated
    first): route and rank every batch, one device plan per rank, every rank's
    scatter into the others' receive buffers, the local experts, and every
    rank's combine from the others' output buffers -- in stream order, which
    orders the phases as the barriers of `forward_p2p` do.  No host wait.
    Returns the G layer outputs."""
    if len(ranks) != len(xs):
        raise ValueError("one batch per rank")
    seg_all = torch.stack([rk.route(x) for rk, x in zip(ranks, xs)])
    for rk in ranks:
        rk.plan(seg_all)
    for rk, x in zip(ranks, xs):
        rk.scatter(x)
    for rk, x in zip(ranks, xs):
        rk.shared(x)
        rk.experts()
    return [rk.combine() for rk in ranks]


def open_peer_buffers(rank_state: PeerRank, group=None) -> None:
    """Across processes (one per GPU, torch.distributed initialised): give the
    rank receive and output buffers other processes can map (CUDA IPC), swap
    handles with every rank, map the peers' and connect the tables.  Release
    with rank_state.release() before the process group is destroyed."""
    import torch.distributed as dist
    k = rank_state.k
    G, rank = dist.get_world_size(group), dist.get_rank(group)
    if G != k.n_ranks or rank != k.rank:
        raise RuntimeError(f"process group rank {rank}/{G} but the experts were placed for {k.rank}/{k.n_ranks}")
    shape = (k.max_local_rows, k.d_model)
    xb, yb = api.IpcBuffer(shape, k.dtype), api.IpcBuffer(shape, k.dtype)
    k.x_loc, k.y_loc = xb.tensor, yb.tensor
    rank_state.ipc = [xb, yb]
    handles = [None] * G
    dist.all_gather_object(handles, (xb.handle(), yb.handle()), group=group)
    recv, out = [], []
    for q, (hx, hy) in enumerate(handles):
        if q == rank:
            recv.append(xb.ptr)
            out.append(yb.ptr)
            continue
        px, py = api.IpcBuffer(shape, k.dtype, handle=hx), api.IpcBuffer(shape, k.dtype, handle=hy)
        rank_state.ipc += [px, py]
        recv.append(px.ptr)
        out.append(py.ptr)
    rank_state.connect(recv, out)


def _stream_barrier(group=None) -> None:
    """Every rank's work enqueued so far has completed before any rank's
    next kernel starts: a one-element all-reduce ordered on the current stream."""
    import torch.distributed as dist
    flag = torch.zeros(1, dtype=torch.float32, device=torch.cuda.current_device())
    dist.all_reduce(flag, group=group)


def forward_p2p(rank_state: PeerRank, x: torch.Tensor, y: torch.Tensor | None = None, group=None) -> torch.Tensor:
    """One expert-parallel forward with the exchange over peer memory
    (open_peer_buffers first).  Per rank: route and rank; all-gather of the
    segment offsets into device memory; device plan; scatter of the kept rows
    into their experts' ranks; barrier; shared and local experts; barrier;
    combine from the ranks that computed the outputs.  The barriers also
    order consecutive forwards: a rank scatters into a peer's receive buffer
    only after that peer's experts have read it, and computes into its output
    buffer only after every peer's combine has read it."""
    import torch.distributed as dist
    k = rank_state.k
    G = dist.get_world_size(group)
    if G != k.n_ranks or dist.get_rank(group) != k.rank:
        raise RuntimeError("the process group does not match the expert placement")
    seg = rank_state.route(x)
    seg_all = torch.empty((G, seg.numel()), dtype=seg.dtype, device=seg.device)
    dist.all_gather_into_tensor(seg_all, seg, group=group)
    rank_state.plan(seg_all)
    rank_state.scatter(x)
    _stream_barrier(group)
    rank_state.shared(x)
    rank_state.experts()
    _stream_barrier(group)
    return rank_state.combine(y)
