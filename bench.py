#!/usr/bin/env python
"""Benchmark of the sparse-MoE FFN layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mixtral] [--impl ours|reference]

One step = one moe_layer_forward (router -> dispatch -> routed SwiGLU experts
-> shared experts -> combine, plus balance statistics) over one batch of T
tokens of seeded synthetic input, weights resident in HBM.  The metric is
tokens per second; for N > 1 (launched with torchrun, one rank per GPU) every
rank runs its own independent batch (no collective on the data path: the layer
does not shard), and value = N * T / (max over ranks of the step time).

Printed (rank 0): one JSON line with the device-timed value, the end-to-end
value through the public API with host buffers (H2D of x and D2H of y and the
statistics inside the timed region), the roofline of the dominant kernel (the
routed up/gate SwiGLU GEMM) timed with CUDA events on its own stream, per-stage
times, SM clocks sampled during the timed region, and the float64 oracle timed
on a bounded sample on the host's cores.

--impl reference times the oracle itself (the CPU reference), a bounded
sample of tokens per step, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_mixture_experts_04_b200 import MoeLayer, api  # noqa: E402
from sparse_mixture_experts_04_b200 import _lib  # noqa: E402
from sparse_mixture_experts_04_b200.synth import CONFIGS, extra_activations, generate  # noqa: E402

METRIC = "MoE layer fwd tokens/s (BF16, 1 B200); expert GEMM % peak; dispatch GB/s"
L2_BYTES = 126 * 1024 * 1024
EP_RANKS = 8  # ranks of the emulated expert-parallel forward
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# oracle tokens per reference step / in the cpu_baseline sample (about 0.5-1 s each)
REF_TOKENS = {"tiny_fp32": 256, "mixtral": 2, "zen_fine": 8, "skewed": 16, "decode": 2}
CPU_SAMPLE_TOKENS = {"tiny_fp32": 2048, "mixtral": 64, "zen_fine": 192, "skewed": 384, "decode": 64}


def workload_desc(cfg) -> str:
    return cfg.description


def activation_batches(cfg) -> tuple[int, int]:
    """Rotating activation batches (count, bytes each): together more than
    twice the L2, so no step finds its input in L2."""
    x_bytes = cfg.T * cfg.d_model * (2 if cfg.dtype == "bf16" else 4)
    return min(max(2, math.ceil(2 * L2_BYTES / x_bytes) + 1), 64), x_bytes


def weight_bytes(cfg) -> int:
    es = 2 if cfg.dtype == "bf16" else 4
    d, F, E, Ns = cfg.d_model, cfg.d_ff, cfg.n_experts, cfg.n_shared
    return es * (E * d + 3 * F * d * (E + Ns))


def config_dict(cfg, world: int) -> dict:
    """The workload's `config` object, the same on both arms."""
    n_x, x_bytes = activation_batches(cfg)
    return {"workload": workload_desc(cfg), "T": cfg.T, "d_model": cfg.d_model, "n_experts": cfg.n_experts,
            "top_k": cfg.top_k, "d_ff": cfg.d_ff, "n_shared": cfg.n_shared,
            "capacity_factor": cfg.capacity_factor, "global_batch": world * cfg.T,
            "parallelism": f"replicas x{world} (independent batch per GPU, no data-path collective)",
            "l2": (f"{n_x} rotating activation batches ({n_x * x_bytes / 2**20:.0f} MiB) and "
                   f"{weight_bytes(cfg) / 2**30:.2f} GiB of weights per step" +
                   ("; both larger than the 126 MB L2, no flush" if weight_bytes(cfg) > L2_BYTES else
                    "; the weights fit in the 126 MB L2 and stay there (a latency-bound layer), no flush"))}


def host_cpu() -> dict:
    """The host's logical core count and CPU model (for the CPU baselines)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    with open(os.path.join(ROOT, "sparse_mixture_experts_04_b200", "csrc", "expert_gemm.cu"), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per launch of the up/gate GEMM from the committed ncu summary,
    or None when absent or taken on an older version of the kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload, {}).get("expert_up_swiglu")
    if not e or e.get("source_sha256_16") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every few ms."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int):
        self.samples, self.power, self.reasons, self.err = [], [], 0, None
        self._stop = threading.Event()
        self.max_mhz = None
        self.match = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid).lower().replace("gpu-", "")
            h = None
            n = pynvml.nvmlDeviceGetCount()
            for i in range(n):
                hi = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(hi)
                u = (u.decode() if isinstance(u, bytes) else u).lower().replace("gpu-", "")
                if u == uuid:
                    h, self.match = hi, f"uuid (nvml index {i} of {n})"
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index if n > 1 else 0)
                self.match = f"index fallback (nvml index {device_index if n > 1 else 0} of {n})"
            self.h = h
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML unavailable: report, do not fail the benchmark
            self.h, self.err = None, f"{type(e).__name__}: {e}"

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
                self.power.append(self.nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0)
            except Exception as e:
                self.err = str(e)
                return
            time.sleep(0.005)

    def __enter__(self):
        if self.h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.h is not None:
            self._t.join()

    def summary(self) -> dict:
        if self.h is None:
            return {"error": self.err}
        names = sorted(n for bit, n in self.REASONS.items() if self.reasons & bit)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(self.samples) if self.samples else None,
                "power_w_max": max(self.power) if self.power else None,
                "reasons": names, "samples": len(self.samples), "device": self.match}

    def rejected(self) -> bool:
        if self.h is None or not self.samples:
            return False
        bad = {"hw_slowdown", "sw_thermal_slowdown", "hw_thermal_slowdown"}
        if bad & set(self.summary()["reasons"]):
            return True
        med = statistics.median(self.samples)
        return self.max_mhz is not None and med < 0.6 * self.max_mhz and not (self.reasons & 0x4)


# ------------------------------------------------------------------ helpers
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    """Maximum of a per-rank scalar (a step time) over all ranks."""
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_config(cfg, rank: int):
    """Each rank runs its own independent batch: seed shifted by the rank."""
    return cfg.replace(seed=cfg.seed + 1000 * rank)


def algorithmic_flops(cfg, kept_pairs: int) -> dict:
    d, F, E, T, Ns = cfg.d_model, cfg.d_ff, cfg.n_experts, cfg.T, cfg.n_shared
    return {"router": 2.0 * T * d * E, "up": 4.0 * d * F * kept_pairs, "down": 2.0 * d * F * kept_pairs,
            "shared": 6.0 * d * F * Ns * T}


def shared_mixed(cfg, prob) -> bool:
    """True when the library runs the shared experts in the routed experts'
    launches (BF16, shared experts, both FFNs on the same tile shape: CTA
    pairs for groups of at least 256 expected rows -- routed T * K / E capped
    by the capacity, shared T -- single CTAs below), so the up and down stages
    cover both."""
    if cfg.dtype != "bf16" or cfg.n_shared == 0 or os.environ.get("MOE_B200_MIX_SHARED", "1") == "0":
        return False
    expected = cfg.T * cfg.top_k // cfg.n_experts
    cap = api.capacity(prob)
    if cap >= 0:
        expected = min(expected, cap)
    return api.max_rows(prob) > 0 and (expected >= 256) == (cfg.T >= 256)


def shared_up_bytes(cfg) -> float:
    """Algorithmic HBM bytes of the shared experts' up/gate projection: their
    W13, x read once and their H written once."""
    es = 2 if cfg.dtype == "bf16" else 4
    d, F, Ns, T = cfg.d_model, cfg.d_ff, cfg.n_shared, cfg.T
    return es * (Ns * 2.0 * F * d + T * d + T * Ns * F)


def up_gemm_bytes(cfg, kept_per_expert) -> float:
    """Algorithmic HBM bytes of the routed up/gate GEMM: the W13 slices of every
    expert that received a row, its x_perm rows read once and H written once."""
    es = 2 if cfg.dtype == "bf16" else 4
    d, F = cfg.d_model, cfg.d_ff
    touched = sum(1 for k in kept_per_expert if k > 0)
    rows = sum(kept_per_expert)
    return es * (touched * 2.0 * F * d + rows * d + rows * F)


def roofline(cfg, flops: float, nbytes: float, launch_ms: float, peaks: dict, peak_src: str, traffic,
             timed_s: float, kernel: str = "routed up/gate GEMM with SwiGLU epilogue (tcgen05)") -> dict:
    """Bound = whichever of tensor time (flops / dense BF16 peak) and HBM time
    (bytes / copy bandwidth) is longer; achieved and peak are in that unit.
    A tensor-bound kernel is compared with the burst GEMM peak when the timed
    region is short (the burst figure is a GEMM timed alone for a moment), and
    with the sustained one (a GEMM run back to back for seconds, under the
    power limit) only when the timed region lasts a second or more; the other
    ratio is reported beside it."""
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    src = "measured (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    r = {"kernel": kernel,
         "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": nbytes, "launch_ms": launch_ms,
         "traffic": traffic}
    if t_tensor >= t_hbm:
        a = flops / (launch_ms * 1e-3) / 1e12
        sus = peaks.get("bf16_tflops_sustained")
        if sus and timed_s >= 1.0:
            r.update(bound="tensor", achieved=a, peak=sus, unit="TFLOP/s", frac=a / sus,
                     peak_source=f"{src} bf16 dense sustained (timed region {timed_s:.2f} s)",
                     frac_of_burst=a / peaks["bf16_tflops"])
        else:
            r.update(bound="tensor", achieved=a, peak=peaks["bf16_tflops"], unit="TFLOP/s",
                     frac=a / peaks["bf16_tflops"],
                     peak_source=f"{src} bf16 dense burst (timed region {timed_s:.3f} s, under a second)")
            if sus:
                r["frac_of_sustained"] = a / sus
    else:
        a = nbytes / (launch_ms * 1e-3) / 1e9
        r.update(bound="hbm", achieved=a, peak=peaks["hbm_gbs"], unit="GB/s",
                 frac=a / peaks["hbm_gbs"], peak_source=f"{src} HBM copy bandwidth")
    return r


def stage_spans(rows) -> dict:
    """Mean per-stage device spans in us from moe_layer_forward_clocked's
    clocks (one row of 2 * NUM_CLOCKS per forward); dispatch+gather runs from
    the dispatch kernels' first start to the gather's last end."""
    names = _lib.CLOCK_NAMES
    acc = {}

    def span(row, a, b):
        s, e = row[2 * names.index(a)] & 0xFFFFFFFFFFFFFFFF, row[2 * names.index(b) + 1] & 0xFFFFFFFFFFFFFFFF
        if s == 0 or e == 0:
            return None
        return (e - ((~s) & 0xFFFFFFFFFFFFFFFF)) / 1e3

    for row in rows:
        vals = {n: span(row, n, n) for n in names}
        vals["dispatch+gather"] = span(row, "dispatch", "gather")
        for k, v in vals.items():
            if v is not None:
                acc.setdefault(k, []).append(v)
    return {k: statistics.mean(v) for k, v in acc.items()}


def dispatch_bytes(cfg, kept_pairs: int) -> float:
    """topk_idx read twice (histogram, rank) + slot_of / perm written + x rows read + x_perm written."""
    es = 2 if cfg.dtype == "bf16" else 4
    TK = cfg.T * cfg.top_k
    return 4.0 * TK * 2 + 4.0 * TK + 4.0 * kept_pairs + 2.0 * kept_pairs * cfg.d_model * es


def router_bytes(cfg) -> float:
    """x read + W_g read + logits written + top-K indices and gates written."""
    es = 2 if cfg.dtype == "bf16" else 4
    T, E, K, d = cfg.T, cfg.n_experts, cfg.top_k, cfg.d_model
    return 1.0 * T * d * es + 1.0 * E * d * es + 4.0 * T * E + 8.0 * T * K


def combine_bytes(cfg, kept_pairs: int) -> float:
    """kept y_perm rows read + y_shared read (if any) + y written + slot_of and gates read."""
    es = 2 if cfg.dtype == "bf16" else 4
    T, K, d = cfg.T, cfg.top_k, cfg.d_model
    shared = 1.0 * T * d * es if cfg.n_shared > 0 else 0.0
    return 1.0 * kept_pairs * d * es + shared + 1.0 * T * d * es + 8.0 * T * K


# ------------------------------------------------------------------ oracle timing
def oracle_tokens_per_s(cfg, inp, n_tokens: int, offset: int = 0):
    """The float64 oracle's full pipeline on n_tokens tokens of the workload
    (gate logits, softmax/top-K, dispatch, SwiGLU experts, combine).  The sample
    is routed as a batch of its own with no capacity limit (so every sampled
    token does its full K experts of work).  Returns (tokens/s, seconds)."""
    import oracle
    from sparse_mixture_experts_04_b200.synth import bf16_bits

    def host_np(t):
        if t is None or isinstance(t, np.ndarray):
            return t
        return bf16_bits(t) if t.dtype == torch.bfloat16 else t.contiguous().numpy()

    rows = (np.arange(n_tokens) + offset) % cfg.T
    x = host_np(inp["x"])[rows]
    t0 = time.perf_counter()
    l = oracle.gate_logits(x, host_np(inp["w_gate"]), inp["logit_offset"])
    idx, w, p = oracle.select(l, cfg.top_k, bias=inp["sel_bias"])
    disp = oracle.dispatch(idx, cfg.n_experts, -1)
    oracle.layer_rows(x, host_np(inp["w13"]), host_np(inp["w2"]), idx, w, disp["slot_of"],
                      w13_shared=host_np(inp.get("w13_shared")), w2_shared=host_np(inp.get("w2_shared")))
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt


def run_reference(args, cfg):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    inp = generate(cfg)
    for i in range(args.warmup):
        oracle_tokens_per_s(cfg, inp, REF_TOKENS[cfg.name], offset=i)
    times = []
    for i in range(args.steps):
        _, dt = oracle_tokens_per_s(cfg, inp, REF_TOKENS[cfg.name], offset=args.warmup + i)
        times.append(dt)
    step_s = sum(times) / len(times)
    value = REF_TOKENS[cfg.name] / step_s
    sample = (f"{REF_TOKENS[cfg.name]} token(s) of the {cfg.name} workload per step through the float64 oracle "
              "(gate logits, top-K, dispatch, SwiGLU experts, combine), one thread")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(cfg, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample,
                             **host_cpu()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def run_ours(args, cfg):
    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    rcfg = rank_config(cfg, rank)
    inp = generate(rcfg)
    layer = MoeLayer.from_inputs(inp)
    T = cfg.T
    n_x, x_bytes = activation_batches(cfg)
    xs_host = [inp["x"]] + extra_activations(rcfg, n_x - 1)
    xs = [x.cuda() for x in xs_host]
    y = torch.empty((T, cfg.d_model), dtype=layer.dtype, device="cuda")
    stream = torch.cuda.current_stream()

    def step(i, events=None):
        if events is None:
            return api.moe_layer_forward(layer.prob, xs[i % n_x], layer.weights, y, layer.routing, layer.stats,
                                         layer.ws, stream)
        return api.moe_layer_forward_profiled(layer.prob, xs[i % n_x], layer.weights, y, layer.routing,
                                              layer.stats, layer.ws, events, stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    status = api.read_device_status(layer.ws)
    if status:
        raise RuntimeError(f"device status {status:#x} after warm-up")

    def make_events(n, which):
        evs = [[torch.cuda.Event(enable_timing=True) if j in which else None for j in range(_lib.NUM_EVENTS)]
               for _ in range(n)]
        for row in evs:       # create the underlying events before they are handed to the library
            for e in row:
                if e is not None:
                    e.record(stream)
        return evs

    UP = (_lib.EVENT_NAMES.index("dispatched"), _lib.EVENT_NAMES.index("up"))

    def timed_region():
        # Inside the timed region only the two events around the dominant kernel
        # (the routed up/gate GEMM) are recorded, so the kernels of a forward
        # otherwise follow each other directly on the stream.
        evs = make_events(args.steps, UP)
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        n_k = 0
        with ClockSampler(local_rank) as clk:
            start.record(stream)
            for i in range(args.steps):
                n_k += step(args.warmup + i, evs[i])
            end.record(stream)
            torch.cuda.synchronize()
        barrier(world)
        ms = start.elapsed_time(end) / args.steps
        up_ms = sum(evs[i][UP[0]].elapsed_time(evs[i][UP[1]]) for i in range(args.steps)) / args.steps
        return ms, up_ms, n_k, clk

    ms, up_ms, n_kernels, clk = timed_region()
    remeasured = False
    if clk.rejected():
        ms, up_ms, n_kernels, clk = timed_region()
        remeasured = True
    ms_max = max_over_ranks(ms, world)
    timed_s = ms_max * args.steps * 1e-3

    # per-stage breakdown: a separate short pass with an event at every stage boundary
    n_prof = min(args.steps, 10)
    evs = make_events(n_prof, set(range(_lib.NUM_EVENTS)))
    for i in range(n_prof):
        step(i, evs[i])
    torch.cuda.synchronize()
    stage = {}
    for j in range(1, _lib.NUM_EVENTS):
        stage[_lib.EVENT_NAMES[j]] = sum(evs[i][j - 1].elapsed_time(evs[i][j]) for i in range(n_prof)) / n_prof

    # device-stamped stage spans (moe_layer_forward_clocked): the forwards run back to
    # back with no events between their kernels; every stage kernel stamps the global
    # timer when it may start reading its inputs (after the programmatic-launch wait)
    # and when its last CTA ends
    n_clk = min(args.steps, 20)
    clocks = torch.zeros((n_clk, 2 * _lib.NUM_CLOCKS), dtype=torch.int64, device="cuda")
    for i in range(n_clk):
        api.moe_layer_forward_clocked(layer.prob, xs[i % n_x], layer.weights, y, layer.routing, layer.stats,
                                      layer.ws, clocks[i], stream)
    torch.cuda.synchronize()
    clock_spans = stage_spans(clocks.cpu().tolist())

    # end to end through the public API (MoeLayer.forward_host): every step copies
    # its x from pinned host memory and its y and statistics back; the copies of
    # neighbouring steps overlap the kernels (separate streams, double buffers).
    xh = [x.pin_memory() for x in xs_host[: min(n_x, 4)]]
    n_e2e = args.steps
    xs_e = [xh[i % len(xh)] for i in range(n_e2e)]
    ys_e = [torch.empty((T, cfg.d_model), dtype=layer.dtype).pin_memory() for _ in range(2)]
    st_e = [torch.empty(layer.stats.numel(), dtype=torch.float32).pin_memory() for _ in range(2)]
    layer.forward_host(xs_e[:2], ys_e, st_e)                       # warm-up
    torch.cuda.synchronize()
    barrier(world)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    layer.forward_host(xs_e, [ys_e[i % 2] for i in range(n_e2e)], [st_e[i % 2] for i in range(n_e2e)])
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end) / n_e2e, world)
    h2d = xs_e[0].numel() * xs_e[0].element_size()
    d2h = ys_e[0].numel() * ys_e[0].element_size() + layer.stats.numel() * 4
    y = torch.empty(0)

    # the same forward replayed from a CUDA graph (MoeLayer.capture): each step copies its
    # batch into the graph's static input and replays; reported beside the metric
    graph = None
    if not args.no_graph:
        layer.capture()
        for i in range(args.warmup):
            layer.forward_graphed(xs[i % n_x])
        torch.cuda.synchronize()
        barrier(world)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for i in range(args.steps):
            layer.forward_graphed(xs[i % n_x])
        g1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        g_ms = max_over_ranks(g0.elapsed_time(g1) / args.steps, world)
        graph = {"ms_per_step": g_ms, "tokens_per_s": world * T / (g_ms * 1e-3),
                 "note": "one CUDA-graph replay of moe_layer_forward per step after a device copy of the "
                         "step's batch into the graph's static input"}
        layer._graph = None

    # training: the backward of a forward over the same batch (moe_layer_backward),
    # timed on its own (not part of the forward metric); BF16 problems only
    bwd = None
    if cfg.dtype == "bf16" and not args.no_backward:
        # a training layer over the same weights: its forward keeps the gate/up projections
        P = layer.prob
        tprob = api.make_problem(P.T, P.d_model, P.n_experts, P.top_k, P.d_ff, P.n_shared, P.capacity_factor,
                                 "bf16", P.flags | api.FLAG_SAVE_GU, P.alpha)
        tlayer = MoeLayer(tprob, layer.weights)
        gen = torch.Generator(device="cuda").manual_seed(rcfg.seed)
        dy = torch.randn((T, cfg.d_model), generator=gen, device="cuda").to(torch.bfloat16)
        n_b = 3
        b_ms = []
        f_ms = []
        for i in range(n_b + 2):
            f0, b0, b1 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            f0.record(stream)
            tlayer.forward(xs[0], stream=stream)
            b0.record(stream)
            tlayer.backward(xs[0], dy, 1.0, 0.0, stream=stream)
            b1.record(stream)
            torch.cuda.synchronize()
            if i >= 2:
                f_ms.append(f0.elapsed_time(b0))
                b_ms.append(b0.elapsed_time(b1))
        if api.read_device_status(tlayer.ws):
            raise RuntimeError("device status after the backward")
        kept_b = int(tlayer.routing["seg_off"][-1].item())
        bflops = 12.0 * cfg.d_model * cfg.d_ff * (kept_b + cfg.n_shared * T) + 4.0 * T * cfg.d_model * cfg.n_experts
        b_tflops = bflops / (statistics.median(b_ms) * 1e-3) / 1e12
        bwd = {"ms": statistics.median(b_ms), "training_forward_ms": statistics.median(f_ms),
               "algorithmic_tflop": bflops / 1e12, "tflops": b_tflops,
               "frac_of_bf16_peak": b_tflops / load_peaks()[0]["bf16_tflops"],
               "note": "moe_layer_backward after a MOE_FLAG_SAVE_GU forward of the same batch (which keeps the "
                       "gate/up projections), median of 3; 12 d F FLOPs per expert row (dh, dx, dW13, dW2) + "
                       "router 4 T d E"}
        del tlayer, dy

    # the expert-parallel forward (experts split over EP_RANKS ranks), emulated on this one GPU:
    # every rank's share of the experts and its own batch, every exchange a device copy
    # (ep.forward_emulated); reported beside the metric, not part of it
    epl = None
    if world == 1 and cfg.dtype == "bf16" and not args.no_ep and cfg.n_experts % EP_RANKS == 0:
        from sparse_mixture_experts_04_b200 import ep
        G = EP_RANKS
        ranks = [ep.EpRank(ep.CudaExperts(layer.prob, ep.split_weights(layer.weights, G, r), G, r)) for r in range(G)]
        xb = [xs[r % n_x] for r in range(G)]
        for _ in range(2):
            ep.forward_emulated(ranks, xb)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_ep = 3
        e0.record(stream)
        for _ in range(n_ep):
            ep.forward_emulated(ranks, xb)
        e1.record(stream)
        torch.cuda.synchronize()
        ep_ms = e0.elapsed_time(e1) / n_ep
        row_bytes = cfg.d_model * 2
        # per rank and direction: its rows going out to other ranks plus the outputs it sends back
        out_rows = [sum(n for p_, o_, n in rk.send.tolist() if p_ != rk.k.rank) +
                    sum(n for p_, o_, n in rk.recv.tolist() if p_ != rk.k.rank) for rk in ranks]
        xbytes = max(out_rows) * row_bytes
        # the same ranks with the exchange inside the kernels (moe_ep_scatter into the experts'
        # ranks' receive buffers, moe_ep_combine from their output buffers, device plan)
        peers = [ep.PeerRank(rk.k) for rk in ranks]
        ep.connect_emulated(peers)
        for _ in range(2):
            ep.forward_emulated_p2p(peers, xb)
        torch.cuda.synchronize()
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record(stream)
        for _ in range(n_ep):
            ep.forward_emulated_p2p(peers, xb)
        p1.record(stream)
        torch.cuda.synchronize()
        p2p_ms = p0.elapsed_time(p1) / n_ep
        del peers
        epl = {"ranks": G, "emulated_on_one_gpu": True, "ms_per_step_all_ranks": ep_ms,
               "peer_memory": {"ms_per_step_all_ranks": p2p_ms, "tokens_per_s_on_one_gpu": G * T / (p2p_ms * 1e-3),
                               "note": "the exchange inside the kernels: rows scattered into the experts' ranks' "
                                       "receive buffers, outputs read back by the combine, plan on the device, no "
                                       "host wait (ep.forward_emulated_p2p)"},
               "tokens_per_step": G * T, "tokens_per_s_on_one_gpu": G * T / (ep_ms * 1e-3),
               "exchange_bytes_per_rank_per_direction_max": xbytes,
               "modelled_exchange_ms_at_770GBps": xbytes / 770e9 * 1e3,
               "note": f"{G} ranks' expert shares and batches run one after another on one GPU through "
                       "ep.forward_emulated (route, dispatch, exchange as device copies, local experts, return, "
                       "combine); includes a device-to-host copy of the segment offsets per step; the NVLink "
                       "time is modelled from the bytes, not measured (one GPU per run)"}
        del ranks

    kept = int(layer.routing["seg_off"][-1].item())
    up_bytes = up_gemm_bytes(cfg, layer.routing["kept"].tolist())
    flops = algorithmic_flops(cfg, kept)
    peaks, peak_src = load_peaks()
    mixed = shared_mixed(cfg, layer.prob)
    gemm_ms = stage["up"] + stage["down"]
    gemm_flops = flops["up"] + flops["down"] + (flops["shared"] if mixed else 0.0)
    gemm_tflops = gemm_flops / (gemm_ms * 1e-3) / 1e12
    if mixed:   # the dominant launch computes the shared experts' up projection too
        roof = roofline(cfg, flops["up"] + 4.0 * cfg.d_model * cfg.d_ff * cfg.n_shared * cfg.T,
                        up_bytes + shared_up_bytes(cfg), up_ms, peaks, peak_src, ncu_traffic(cfg.name),
                        timed_s, kernel="routed + shared up/gate GEMM with SwiGLU epilogue, one launch (tcgen05)")
    else:
        roof = roofline(cfg, flops["up"], up_bytes, up_ms, peaks, peak_src, ncu_traffic(cfg.name), timed_s)
    # HBM fractions of the memory-bound stages from the device-stamped spans
    # (first CTA start to last CTA end of the stage's kernels), and from the
    # event pass beside them (which adds a launch gap at every stage boundary)
    mem_bytes = {"router": router_bytes(cfg), "dispatch": dispatch_bytes(cfg, kept),
                 "combine": combine_bytes(cfg, kept)}
    span_key = {"router": "route", "dispatch": "dispatch+gather", "combine": "combine"}
    event_key = {"router": "routed", "dispatch": "dispatched", "combine": "end"}
    gbs_clock = {k: (mem_bytes[k] / (clock_spans[span_key[k]] * 1e-6) / 1e9
                     if clock_spans.get(span_key[k]) else None) for k in mem_bytes}
    gbs_event = {k: mem_bytes[k] / (stage[event_key[k]] * 1e-3) / 1e9 for k in mem_bytes}
    disp_gbs = gbs_clock["dispatch"] or gbs_event["dispatch"]
    router_gbs = gbs_clock["router"] or gbs_event["router"]
    combine_gbs = gbs_clock["combine"] or gbs_event["combine"]
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        n = CPU_SAMPLE_TOKENS[cfg.name]
        v, dt = oracle_tokens_per_s(cfg, inp, n)
        cpu = {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": f"{n} tokens of the {cfg.name} workload through the float64 oracle's full pipeline "
                         f"(no capacity limit within the sample), one thread, {dt:.1f} s", **host_cpu()}
        # the same source built with OpenMP on every host core (same bits; a second baseline)
        import oracle
        cores = oracle.set_threads(os.cpu_count() or 1)
        try:
            n_omp = n * cores
            v_omp, dt_omp = oracle_tokens_per_s(cfg, inp, n_omp)
        finally:
            oracle.set_threads(1)
        cpu["openmp"] = {"value": v_omp, "unit": "tokens/s", "cores": cores,
                         "sample": f"{n_omp} tokens, the oracle built with -fopenmp (gate logits and layer rows "
                                   f"split over {cores} threads), {dt_omp:.1f} s"}
    total_flops = sum(flops.values())
    line = {
        "metric": METRIC, "value": world * T / (ms_max * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
        "data": "synthetic: seeded N(0,1) activations, random-init N(0,1/d_in) weights",
        "config": config_dict(cfg, world),
        "e2e": {"value": world * T / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "roofline": roof,
        "cpu_baseline": cpu,
        "gpu_launches": n_kernels,
        "clocks": {**clk.summary(), "remeasured": remeasured},
        "stages_ms": stage,
        "stages_note": "separate pass with an event at every stage boundary" +
                       ("; the shared experts run in the up and down launches (the shared stage is empty)"
                        if mixed else ""),
        "kept_pairs": kept, "dropped_pairs": cfg.T * cfg.top_k - kept,
        "expert_gemm_tflops": gemm_tflops, "expert_gemm_pct_peak": 100.0 * gemm_tflops / peaks["bf16_tflops"],
        "expert_gemm_pct_sustained_peak": (100.0 * gemm_tflops / peaks["bf16_tflops_sustained"]
                                           if peaks.get("bf16_tflops_sustained") else None),
        "dispatch_gbs": disp_gbs, "router_gbs": router_gbs, "combine_gbs": combine_gbs,
        "hbm_frac": {"router": router_gbs / peaks["hbm_gbs"], "dispatch": disp_gbs / peaks["hbm_gbs"],
                     "combine": combine_gbs / peaks["hbm_gbs"],
                     "note": "algorithmic bytes / the stage's device-stamped span (moe_layer_forward_clocked: "
                             "first CTA start to last CTA end of the stage's kernels, dispatch = scan+rank "
                             "start to gather end, mean of back-to-back forwards) / the measured HBM copy "
                             "bandwidth"},
        "stage_clock_us": clock_spans,
        "hbm_frac_event_stages": {k: gbs_event[k] / peaks["hbm_gbs"] for k in gbs_event},
        "layer_tflops": total_flops / (ms * 1e-3) / 1e12,
        "backward": bwd,
        "expert_parallel": epl,
        "graph": graph,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="mixtral", choices=list(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip the (separately reported) backward timing")
    ap.add_argument("--no-ep", action="store_true", help="skip the (separately reported) emulated expert-parallel timing")
    ap.add_argument("--no-graph", action="store_true", help="skip the (separately reported) CUDA-graph replay timing")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)   # at least 3 untimed warm-up steps, always
    cfg = CONFIGS[args.workload]
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
