"""Python binding of the C ABI, with the same entry-point names.

Argument marshalling only: every function passes torch device tensors' data
pointers (and the current CUDA stream) to libmoe_b200.so and raises MoeError
on a non-zero status.  No step of the layer is computed here.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import (BIAS_UPDATE_PROPORTIONAL, BIAS_UPDATE_SIGN, DTYPE_BF16, DTYPE_F32, EXTENDED_STATS, FFN_ROUTED,
                   FFN_SHARED, FLAG_BIAS_LOGIT, FLAG_EXPERT_CAPACITY, FLAG_EXTENDED_STATS, FLAG_LOGITS_GIVEN,
                   FLAG_SAVE_GU,
                   MoeError, MoeGrads, MoeProblem, MoeRouting, MoeWeights)

__all__ = ["MoeError", "MoeProblem", "make_problem", "workspace_size", "capacity", "max_rows", "alloc_workspace",
           "moe_route", "moe_dispatch", "moe_expert_ffn", "moe_expert_ffn_segments", "moe_combine", "moe_layer_forward",
           "moe_layer_forward_profiled", "moe_layer_forward_clocked", "stage_clock_us", "moe_dispatch_noalloc", "moe_dispatch_capacity", "moe_balance_update",
           "moe_layer_backward", "backward_workspace_size", "alloc_backward_workspace", "moe_ep_plan",
           "reset_device_status", "read_device_status", "FLAG_LOGITS_GIVEN", "FLAG_BIAS_LOGIT",
           "FLAG_EXTENDED_STATS", "FLAG_EXPERT_CAPACITY", "FLAG_SAVE_GU", "EXTENDED_STATS", "stats_size",
           "BIAS_UPDATE_SIGN", "BIAS_UPDATE_PROPORTIONAL",
           "FFN_ROUTED", "FFN_SHARED", "DTYPE_BF16", "DTYPE_F32"]


def make_problem(T, d_model, n_experts, top_k, d_ff, n_shared=0, capacity_factor=0.0, dtype="bf16", flags=0,
                 alpha=0.01) -> MoeProblem:
    dt = {"bf16": DTYPE_BF16, "f32": DTYPE_F32, DTYPE_BF16: DTYPE_BF16, DTYPE_F32: DTYPE_F32}[dtype]
    return MoeProblem(int(T), int(d_model), int(n_experts), int(top_k), int(n_shared), int(d_ff),
                      float(capacity_factor), dt, int(flags), float(alpha))


def _p(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def stats_size(prob: MoeProblem) -> int:
    """Entries of the stats array: 2E+1, or 2E+7 with FLAG_EXTENDED_STATS."""
    return 2 * prob.n_experts + (7 if prob.flags & FLAG_EXTENDED_STATS else 1)


def workspace_size(prob: MoeProblem) -> int:
    n = ctypes.c_size_t(0)
    _lib.check("moe_workspace_size", _lib.lib().moe_workspace_size(ctypes.byref(prob), ctypes.byref(n)))
    return int(n.value)


def capacity(prob: MoeProblem) -> int:
    return int(_lib.lib().moe_capacity(ctypes.byref(prob)))


def max_rows(prob: MoeProblem) -> int:
    return int(_lib.lib().moe_max_rows(ctypes.byref(prob)))


def alloc_workspace(prob: MoeProblem, device="cuda") -> torch.Tensor:
    """A caller-owned workspace (torch's allocator returns 256-byte aligned
    blocks), zero-filled once so that its device status word starts clean."""
    return torch.zeros(workspace_size(prob), dtype=torch.uint8, device=device)


def reset_device_status(ws: torch.Tensor, stream=None) -> None:
    _lib.check("moe_reset_device_status", _lib.lib().moe_reset_device_status(_p(ws), _stream(stream)))


def read_device_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronises the stream; returns the device status bits (0 = clean)."""
    bits = ctypes.c_uint32(0)
    rc = _lib.lib().moe_read_device_status(_p(ws), _stream(stream), ctypes.byref(bits))
    if rc not in (0, -4):
        raise MoeError("moe_read_device_status", rc)
    return int(bits.value)


def moe_route(prob, x, w_gate, logit_offset, sel_bias, logits, topk_idx, topk_w, stats, ws, stream=None):
    rc = _lib.lib().moe_route(ctypes.byref(prob), _p(x), _p(w_gate), _p(logit_offset), _p(sel_bias), _p(logits),
                              _p(topk_idx), _p(topk_w), _p(stats), _p(ws), ws.numel(), _stream(stream))
    _lib.check("moe_route", rc)


def moe_dispatch(prob, topk_idx, x, counts, kept, seg_off, slot_of, perm, x_perm, ws, stream=None):
    rc = _lib.lib().moe_dispatch(ctypes.byref(prob), _p(topk_idx), _p(x), _p(counts), _p(kept), _p(seg_off),
                                 _p(slot_of), _p(perm), _p(x_perm), _p(ws), ws.numel(), _stream(stream))
    _lib.check("moe_dispatch", rc)


def moe_dispatch_noalloc(prob, topk_idx, x, counts, kept, seg_off, slot_of, perm, x_perm, stream=None):
    """moe_dispatch without a workspace, for callers that cannot provide device
    scratch memory (the library's own fixed array is used; see the header)."""
    rc = _lib.lib().moe_dispatch_noalloc(ctypes.byref(prob), _p(topk_idx), _p(x), _p(counts), _p(kept),
                                         _p(seg_off), _p(slot_of), _p(perm), _p(x_perm), _stream(stream))
    _lib.check("moe_dispatch_noalloc", rc)


def moe_dispatch_capacity(prob, topk_idx, expert_capacity, x, counts, kept, seg_off, slot_of, perm, x_perm, ws,
                          stream=None):
    rc = _lib.lib().moe_dispatch_capacity(ctypes.byref(prob), _p(topk_idx), _p(expert_capacity), _p(x), _p(counts),
                                          _p(kept), _p(seg_off), _p(slot_of), _p(perm), _p(x_perm), _p(ws),
                                          ws.numel(), _stream(stream))
    _lib.check("moe_dispatch_capacity", rc)


def moe_balance_update(prob, counts, sel_bias=None, bias_rate=0.0, bias_mode=BIAS_UPDATE_SIGN, count_hist=None,
                       step=0, c_base=1.0, gamma=0.0, expert_capacity=None, stream=None):
    """Selection-bias update and/or adaptive per-expert capacity from one step's
    counts (see moe_balance_update in the header); count_hist [W, E] int32."""
    hist_len = 0 if count_hist is None else int(count_hist.shape[0])
    rc = _lib.lib().moe_balance_update(ctypes.byref(prob), _p(counts), _p(sel_bias), float(bias_rate), int(bias_mode),
                                       _p(count_hist), hist_len, int(step), float(c_base), float(gamma),
                                       _p(expert_capacity), _stream(stream))
    _lib.check("moe_balance_update", rc)


def moe_expert_ffn(prob, mode, x_rows, n_rows, seg_off, w13, w2, y_rows, ws, stream=None):
    rc = _lib.lib().moe_expert_ffn(ctypes.byref(prob), int(mode), _p(x_rows), int(n_rows), _p(seg_off), _p(w13),
                                   _p(w2), _p(y_rows), _p(ws), ws.numel(), _stream(stream))
    _lib.check("moe_expert_ffn", rc)


def moe_expert_ffn_segments(prob, x_rows, n_rows, seg_off, n_segments, w13, w2, y_rows, ws, stream=None):
    """Routed experts over n_segments row segments; segment i uses expert i % E."""
    _lib.check("moe_expert_ffn_segments",
               _lib.lib().moe_expert_ffn_segments(ctypes.byref(prob), _p(x_rows), int(n_rows), _p(seg_off),
                                                  int(n_segments), _p(w13), _p(w2), _p(y_rows), _p(ws), ws.numel(),
                                                  _stream(stream)))


def moe_combine(prob, y_perm, slot_of, topk_w, y_shared, y, ws, stream=None):
    rc = _lib.lib().moe_combine(ctypes.byref(prob), _p(y_perm), _p(slot_of), _p(topk_w), _p(y_shared), _p(y),
                                _p(ws), ws.numel(), _stream(stream))
    _lib.check("moe_combine", rc)


def _weights_struct(w: dict) -> MoeWeights:
    return MoeWeights(_p(w.get("w_gate")), _p(w.get("logit_offset")), _p(w.get("sel_bias")), _p(w["w13"]),
                      _p(w["w2"]), _p(w.get("w13_shared")), _p(w.get("w2_shared")), _p(w.get("expert_capacity")))


def _routing_struct(r: dict | None) -> MoeRouting | None:
    if r is None:
        return None
    return MoeRouting(_p(r.get("logits")), _p(r.get("topk_idx")), _p(r.get("topk_w")), _p(r.get("counts")),
                      _p(r.get("kept")), _p(r.get("seg_off")), _p(r.get("slot_of")), _p(r.get("perm")))


def moe_layer_forward(prob, x, weights: dict, y, routing: dict | None, stats, ws, stream=None):
    w = _weights_struct(weights)
    r = _routing_struct(routing)
    rc = _lib.lib().moe_layer_forward(ctypes.byref(prob), _p(x), ctypes.byref(w), _p(y),
                                      ctypes.byref(r) if r is not None else None, _p(stats), _p(ws), ws.numel(),
                                      _stream(stream))
    _lib.check("moe_layer_forward", rc)


def moe_layer_forward_profiled(prob, x, weights: dict, y, routing: dict | None, stats, ws, events, stream=None) -> int:
    """moe_layer_forward that also records `events` (7 torch.cuda.Event, or None
    entries) at the stage boundaries; returns the number of kernels enqueued."""
    w = _weights_struct(weights)
    r = _routing_struct(routing)
    handles = (ctypes.c_void_p * _lib.NUM_EVENTS)()
    for i, ev in enumerate(events):
        handles[i] = None if ev is None else ev.cuda_event
    n = ctypes.c_int32(0)
    rc = _lib.lib().moe_layer_forward_profiled(ctypes.byref(prob), _p(x), ctypes.byref(w), _p(y),
                                               ctypes.byref(r) if r is not None else None, _p(stats), _p(ws),
                                               ws.numel(), _stream(stream), handles, ctypes.byref(n))
    _lib.check("moe_layer_forward_profiled", rc)
    return int(n.value)


def moe_layer_forward_clocked(prob, x, weights: dict, y, routing: dict | None, stats, ws, clocks, stream=None):
    """moe_layer_forward with device stage clocks: `clocks` is a zero-filled
    int64 device tensor of 2 * NUM_CLOCKS entries (see stage_clock_us)."""
    assert clocks.dtype == torch.int64 and clocks.numel() >= 2 * _lib.NUM_CLOCKS and clocks.is_cuda
    w = _weights_struct(weights)
    r = _routing_struct(routing)
    rc = _lib.lib().moe_layer_forward_clocked(ctypes.byref(prob), _p(x), ctypes.byref(w), _p(y),
                                              ctypes.byref(r) if r is not None else None, _p(stats), _p(ws),
                                              ws.numel(), _stream(stream), _p(clocks))
    _lib.check("moe_layer_forward_clocked", rc)


def stage_clock_us(clocks) -> dict:
    """Per-stage device time in us from one forward's clocks (host copy, any
    integer sequence of 2 * NUM_CLOCKS): end - start for each stage that
    stamped, None for the others."""
    out = {}
    vals = [int(v) & 0xFFFFFFFFFFFFFFFF for v in clocks]
    for s, name in enumerate(_lib.CLOCK_NAMES):
        start_c, end = vals[2 * s], vals[2 * s + 1]
        if start_c == 0 or end == 0:
            out[name] = None
            continue
        start = (~start_c) & 0xFFFFFFFFFFFFFFFF
        out[name] = (end - start) / 1e3
    return out


def backward_workspace_size(prob: MoeProblem) -> int:
    n = ctypes.c_size_t(0)
    _lib.check("moe_backward_workspace_size", _lib.lib().moe_backward_workspace_size(ctypes.byref(prob), ctypes.byref(n)))
    return int(n.value)


def alloc_backward_workspace(prob: MoeProblem, device="cuda") -> torch.Tensor:
    return torch.zeros(backward_workspace_size(prob), dtype=torch.uint8, device=device)


def moe_layer_backward(prob, x, weights: dict, routing: dict | None, fwd_ws, dy, d_loss, d_zloss, grads: dict, ws,
                       stream=None):
    """Gradients of the layer (see moe_layer_backward in the header); grads maps
    dx, dw13, dw2, dw13_shared, dw2_shared, dw_gate, d_offset, d_logits to
    tensors (missing or None: not computed; dw13 and dw2 required)."""
    g = MoeGrads(*[_p(grads.get(k)) for k in ("dx", "dw13", "dw2", "dw13_shared", "dw2_shared", "dw_gate",
                                               "d_offset", "d_logits")])
    r = _routing_struct(routing)
    rc = _lib.lib().moe_layer_backward(ctypes.byref(prob), _p(x), ctypes.byref(_weights_struct(weights)),
                                       ctypes.byref(r) if r is not None else None, _p(fwd_ws), fwd_ws.numel(),
                                       _p(dy), float(d_loss), float(d_zloss), ctypes.byref(g), _p(ws), ws.numel(),
                                       _stream(stream))
    _lib.check("moe_layer_backward", rc)


def moe_ep_plan(n_ranks: int, rank: int, n_experts: int, seg_off_all) -> tuple:
    """Expert-parallel exchange plan (host function, no device).  seg_off_all
    [n_ranks, E+1] int32 (CPU) -> (send [G, 3], recv [G, 3],
    local_seg_off [G*E_l+1]) int32 CPU tensors; see include/moe_b200.h."""
    so = torch.as_tensor(seg_off_all, dtype=torch.int32).contiguous()
    if so.device.type != "cpu":
        raise ValueError("moe_ep_plan takes host (CPU) segment offsets")
    G, E = int(n_ranks), int(n_experts)
    El = E // G if G > 0 else 0
    send = torch.empty((max(G, 1), 3), dtype=torch.int32)
    recv = torch.empty((max(G, 1), 3), dtype=torch.int32)
    local = torch.empty(G * El + 1, dtype=torch.int32)
    if so.numel() != G * (E + 1):
        raise ValueError(f"seg_off_all has {so.numel()} entries, expected {G}x{E + 1}")
    rc = _lib.lib().moe_ep_plan(G, int(rank), E, so.data_ptr(), send.data_ptr(), recv.data_ptr(), local.data_ptr())
    _lib.check("moe_ep_plan", rc)
    return send[:G], recv[:G], local


# ----------------------------------------------------- expert parallel over peer memory
IPC_HANDLE_BYTES = 64


def moe_ep_peer_plan(n_ranks: int, rank: int, n_experts: int, seg_off_all, delta, local_seg_off, stream=None):
    """Device plan of the peer-memory exchange (one kernel, no host wait):
    seg_off_all [G, E+1] int32 (device) -> delta [E] int64 and
    local_seg_off [E/G + 1] int32 (device); see include/moe_b200.h."""
    rc = _lib.lib().moe_ep_peer_plan(int(n_ranks), int(rank), int(n_experts), _p(seg_off_all), _p(delta),
                                     _p(local_seg_off), _stream(stream))
    _lib.check("moe_ep_peer_plan", rc)


def moe_ep_scatter(prob, n_ranks: int, x, perm, seg_off, recv_bufs, delta, stream=None):
    """Each kept row of this rank written into the receive buffer of its
    expert's rank; recv_bufs: [G] int64 device tensor of device pointers."""
    rc = _lib.lib().moe_ep_scatter(ctypes.byref(prob), int(n_ranks), _p(x), _p(perm), _p(seg_off), _p(recv_bufs),
                                   _p(delta), _stream(stream))
    _lib.check("moe_ep_scatter", rc)


def moe_ep_combine(prob, n_ranks: int, out_bufs, delta, topk_idx, slot_of, topk_w, y_shared, y, stream=None):
    """moe_combine reading each kept pair's output from its expert's rank;
    out_bufs: [G] int64 device tensor of device pointers."""
    rc = _lib.lib().moe_ep_combine(ctypes.byref(prob), int(n_ranks), _p(out_bufs), _p(delta), _p(topk_idx),
                                   _p(slot_of), _p(topk_w), _p(y_shared), _p(y), _stream(stream))
    _lib.check("moe_ep_combine", rc)


class IpcBuffer:
    """A whole device allocation (moe_ipc_malloc) another process can map,
    or the mapping of one (moe_ipc_open); `tensor` views it as a torch tensor
    (through __cuda_array_interface__).  release() frees / unmaps it."""

    def __init__(self, shape, dtype, handle: bytes | None = None):
        self.shape, self.dtype = tuple(int(n) for n in shape), dtype
        nbytes = max(1, int(torch.tensor([], dtype=dtype).element_size()))
        for n in self.shape:
            nbytes *= n
        ptr = ctypes.c_void_p()
        if handle is None:
            _lib.check("moe_ipc_malloc", _lib.lib().moe_ipc_malloc(max(nbytes, 16), ctypes.byref(ptr)))
            self.opened = False
        else:
            buf = ctypes.create_string_buffer(bytes(handle), IPC_HANDLE_BYTES)
            _lib.check("moe_ipc_open", _lib.lib().moe_ipc_open(buf, ctypes.byref(ptr)))
            self.opened = True
        self.ptr = int(ptr.value)
        # BF16 has no array-interface type code: viewed as int16, then as BF16
        typestr = {torch.bfloat16: "<i2", torch.float32: "<f4", torch.int32: "<i4", torch.int64: "<i8"}[dtype]
        t = torch.as_tensor(_Iface(self.shape, typestr, self.ptr), device="cuda")
        self.tensor = t.view(torch.bfloat16) if dtype == torch.bfloat16 else t

    def handle(self) -> bytes:
        buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
        _lib.check("moe_ipc_handle", _lib.lib().moe_ipc_handle(self.ptr, buf))
        return buf.raw

    def release(self) -> None:
        if self.ptr:
            self.tensor = None
            fn = _lib.lib().moe_ipc_close if self.opened else _lib.lib().moe_ipc_free
            _lib.check("moe_ipc_release", fn(self.ptr))
            self.ptr = 0


class _Iface:
    def __init__(self, shape, typestr, ptr):
        self.__cuda_array_interface__ = {"shape": shape, "typestr": typestr, "data": (ptr, False), "version": 3,
                                         "strides": None}
