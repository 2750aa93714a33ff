"""MoeLayer: one layer's weights, workspace and routing buffers on the device,
with forward() = one moe_layer_forward call, and forward_host() for batches
that live in (pinned) host memory.  Allocation (through torch), stream
bookkeeping and argument marshalling only."""
from __future__ import annotations

import torch

from . import api


class MoeLayer:
    def __init__(self, prob: api.MoeProblem, weights: dict, device="cuda", keep_routing: bool = True):
        self.prob = prob
        self.device = torch.device(device)
        self.weights = weights
        self.ws = api.alloc_workspace(prob, self.device)
        self.dtype = torch.bfloat16 if prob.dtype == api.DTYPE_BF16 else torch.float32
        T, E, K = prob.T, prob.n_experts, prob.top_k
        self.routing = None
        if keep_routing:
            i32 = dict(dtype=torch.int32, device=self.device)
            self.routing = dict(
                logits=torch.empty((T, E), dtype=torch.float32, device=self.device),
                topk_idx=torch.empty((T, K), **i32), topk_w=torch.empty((T, K), dtype=torch.float32, device=self.device),
                counts=torch.empty(E, **i32), kept=torch.empty(E, **i32), seg_off=torch.empty(E + 1, **i32),
                slot_of=torch.empty((T, K), **i32), perm=torch.empty(max(api.max_rows(prob), 1), **i32))
        self.stats = torch.empty(api.stats_size(prob), dtype=torch.float32, device=self.device)
        if prob.flags & api.FLAG_EXPERT_CAPACITY and weights.get("expert_capacity") is None:
            # start from the uniform capacity (no limit: -1)
            cap = api.capacity(prob)
            cap = -1 if cap < 0 else min(cap, T)
            weights["expert_capacity"] = torch.full((E,), cap, dtype=torch.int32, device=self.device)
        self._balance_step = 0
        self._count_hist = None

    @classmethod
    def from_inputs(cls, inputs: dict, device="cuda", flags: int = 0, keep_routing: bool = True) -> "MoeLayer":
        """Build from synth.generate() output (CPU tensors are copied to the device)."""
        cfg = inputs["cfg"]
        prob = api.make_problem(cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff, cfg.n_shared,
                                cfg.capacity_factor, cfg.dtype, flags, cfg.alpha)
        dev = torch.device(device)

        def to_dev(v):
            if v is None:
                return None
            t = torch.as_tensor(v)
            return t.to(dev).contiguous()

        w = {k: to_dev(inputs.get(k)) for k in ("w_gate", "w13", "w2", "w13_shared", "w2_shared")}
        w["sel_bias"] = to_dev(inputs.get("sel_bias"))
        w["logit_offset"] = to_dev(inputs.get("logit_offset"))
        return cls(prob, w, dev, keep_routing)

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, with_stats: bool = True,
                stream=None) -> torch.Tensor:
        if y is None:
            y = torch.empty((self.prob.T, self.prob.d_model), dtype=self.dtype, device=self.device)
        api.moe_layer_forward(self.prob, x, self.weights, y, self.routing, self.stats if with_stats else None,
                              self.ws, stream)
        return y

    __call__ = forward

    def capture(self, with_stats: bool = True) -> None:
        """Capture one forward into a CUDA graph over static input/output
        buffers (self.graph_x, self.graph_y); forward_graphed() replays it.  The
        layer's launches (memset, kernels with programmatic dependent launch)
        become one graph, so a replay costs one launch on the host.  One eager
        forward runs first, outside the capture, to set the kernels' per-device
        attributes."""
        T, d = self.prob.T, self.prob.d_model
        self.graph_x = torch.zeros((T, d), dtype=self.dtype, device=self.device)
        self.graph_y = torch.empty((T, d), dtype=self.dtype, device=self.device)
        self.forward(self.graph_x, self.graph_y, with_stats)
        torch.cuda.synchronize(self.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            api.moe_layer_forward(self.prob, self.graph_x, self.weights, self.graph_y, self.routing,
                                  self.stats if with_stats else None, self.ws)
        self._graph = g

    def forward_graphed(self, x: torch.Tensor | None = None) -> torch.Tensor:
        """Replay the captured forward (capture() first) on the current stream;
        x (if given) is copied into the static input first.  Returns the static
        output buffer, overwritten by the next replay."""
        if getattr(self, "_graph", None) is None:
            raise RuntimeError("MoeLayer.capture() has not been called")
        if x is not None:
            self.graph_x.copy_(x)
        self._graph.replay()
        return self.graph_y

    def backward(self, x: torch.Tensor, dy: torch.Tensor, d_loss: float = 1.0, d_zloss: float = 0.0,
                 stream=None) -> dict:
        """Gradients of the last forward (same x; the workspace untouched since),
        for dJ/dy = dy and dJ/d(balance loss) = d_loss, dJ/d(z-loss) = d_zloss.
        Returns FP32 weight gradients and dx (activation dtype)."""
        P, dev = self.prob, self.device
        f32 = dict(dtype=torch.float32, device=dev)
        E, d, F, Ns, T = P.n_experts, P.d_model, P.d_ff, P.n_shared, P.T
        g = dict(dx=torch.empty((T, d), dtype=self.dtype, device=dev), dw13=torch.empty((E, 2 * F, d), **f32),
                 dw2=torch.empty((E, d, F), **f32), d_offset=torch.empty(E, **f32),
                 d_logits=torch.empty((T, E), **f32))
        if not P.flags & api.FLAG_LOGITS_GIVEN:
            g["dw_gate"] = torch.empty((E, d), **f32)
        if Ns:
            g["dw13_shared"] = torch.empty((Ns, 2 * F, d), **f32)
            g["dw2_shared"] = torch.empty((Ns, d, F), **f32)
        if getattr(self, "_bwd_ws", None) is None:
            self._bwd_ws = api.alloc_backward_workspace(P, dev)
        api.moe_layer_backward(P, x, self.weights, self.routing, self.ws, dy, d_loss, d_zloss, g, self._bwd_ws,
                               stream)
        return g

    def balance_update(self, bias_rate: float = 0.0, bias_mode: int = api.BIAS_UPDATE_SIGN, c_base: float | None = None,
                       gamma: float = 0.0, window: int = 8, stream=None) -> None:
        """Between steps: move the selection bias against the last forward's
        load (when the layer has one and bias_rate != 0) and, for a layer built
        with FLAG_EXPERT_CAPACITY, set the next forward's per-expert capacities
        from the last `window` forwards' loads (c_base defaults to the
        problem's capacity factor).  One kernel on the stream."""
        if self.routing is None:
            raise ValueError("balance_update needs the routing outputs (keep_routing=True)")
        bias = self.weights.get("sel_bias") if bias_rate != 0.0 else None
        caps = self.weights.get("expert_capacity") if self.prob.flags & api.FLAG_EXPERT_CAPACITY else None
        if bias is None and caps is None:
            return
        hist = None
        if caps is not None:
            if self._count_hist is None or self._count_hist.shape[0] != window:
                self._count_hist = torch.zeros((window, self.prob.n_experts), dtype=torch.int32, device=self.device)
                self._balance_step = 0
            hist = self._count_hist
        cb = self.prob.capacity_factor if c_base is None else c_base
        api.moe_balance_update(self.prob, self.routing["counts"], bias, bias_rate, bias_mode, hist,
                               self._balance_step, cb, gamma, caps, stream)
        if caps is not None:
            self._balance_step += 1

    def forward_host(self, xs_host, ys_host, stats_host=None, stream=None):
        """Run one layer forward per host batch: xs_host[i] [T, d] -> ys_host[i].

        Host tensors should be pinned.  The host->device copy of batch i+1 and
        the device->host copy of batch i-1 run on their own streams while batch
        i computes (two device buffers each for x and y), so the copy engines
        overlap the kernels.  stats_host[i] (optional) receives the [2E+1]
        statistics of batch i.  Returns after every copy has landed."""
        n = len(xs_host)
        if n == 0:
            return
        dev = self.device
        comp = stream if stream is not None else torch.cuda.current_stream(dev)
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        T, d = self.prob.T, self.prob.d_model
        xb = [torch.empty((T, d), dtype=self.dtype, device=dev) for _ in range(2)]
        yb = [torch.empty((T, d), dtype=self.dtype, device=dev) for _ in range(2)]
        sb = [torch.empty_like(self.stats) for _ in range(2)]
        ev = lambda: torch.cuda.Event()
        copied_in = [ev() for _ in range(n)]
        computed = [ev() for _ in range(n)]
        copied_out = [ev() for _ in range(n)]
        h2d.wait_stream(comp)
        d2h.wait_stream(comp)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(h2d):
                if i >= 2:
                    h2d.wait_event(computed[i - 2])       # x buffer b is free again
                xb[b].copy_(xs_host[i], non_blocking=True)
                copied_in[i].record(h2d)
            comp.wait_event(copied_in[i])
            if i >= 2:
                comp.wait_event(copied_out[i - 2])        # y / stats buffers b are free again
            api.moe_layer_forward(self.prob, xb[b], self.weights, yb[b], self.routing, sb[b], self.ws, comp)
            computed[i].record(comp)
            with torch.cuda.stream(d2h):
                d2h.wait_event(computed[i])
                ys_host[i].copy_(yb[b], non_blocking=True)
                if stats_host is not None:
                    stats_host[i].copy_(sb[b], non_blocking=True)
                copied_out[i].record(d2h)
        comp.wait_stream(d2h)
        comp.synchronize()
