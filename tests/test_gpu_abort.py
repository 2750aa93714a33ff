"""The bounded-wait abort path of the tcgen05 kernels, on the GPU.

Every pipeline wait of the fused router and of the single-CTA expert GEMM is
bounded; when one runs out the kernel records MOE_DEV_WAIT_TIMEOUT in the
status word, lets the copies and MMAs it started complete, frees its tensor
memory and returns, so that the stream and the context stay usable.  The test
hook MOE_B200_TEST_STALL_NS makes the MMA thread of those kernels wait for a
barrier phase that nothing completes (for that long), which drives exactly
that path: no fault, trap or endless wait is involved.  After it, a normal
call in the same process must give the oracle's result."""
import time

import numpy as np
import pytest
import torch

import oracle
from helpers import dev, host_np, rel_err
from sparse_mixture_experts_04_b200 import api
from sparse_mixture_experts_04_b200._lib import DEV_WAIT_TIMEOUT
from sparse_mixture_experts_04_b200.synth import exact_router_inputs

pytestmark = pytest.mark.gpu

STALL_NS = "2000000"   # 2 ms instead of the 2 s limit of a real wait


def _route(prob, inp, T, E, K):
    ws = api.alloc_workspace(prob)
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    stats = torch.empty(api.stats_size(prob), dtype=torch.float32, device="cuda")
    api.reset_device_status(ws)
    api.moe_route(prob, dev(inp["x"]), dev(inp["w_gate"]), dev(inp["logit_offset"]), None, logits, idx, w, stats, ws)
    t0 = time.monotonic()
    bits = api.read_device_status(ws)    # synchronises the stream
    return bits, time.monotonic() - t0, idx.cpu().numpy(), w.cpu().numpy()


def test_fused_router_wait_timeout_is_reported_and_the_context_stays_usable(monkeypatch):
    T, d, E, K = 300, 512, 16, 2   # a cluster split of the reduction: several CTAs per tile
    inp = exact_router_inputs(T, d, E, seed=41)
    prob = api.make_problem(T, d, E, K, 64, 0, 1.0, "bf16")
    monkeypatch.setenv("MOE_B200_TEST_STALL_NS", STALL_NS)
    bits, waited, _, _ = _route(prob, inp, T, E, K)
    assert bits & DEV_WAIT_TIMEOUT, f"status {bits:#x}"
    assert waited < 10.0
    monkeypatch.delenv("MOE_B200_TEST_STALL_NS")
    bits, _, idx, w = _route(prob, inp, T, E, K)
    assert bits == 0
    l64 = oracle.gate_logits(host_np(inp["x"]), host_np(inp["w_gate"]), inp["logit_offset"])
    r_idx, r_w, _ = oracle.select(l64, K)
    assert (idx == r_idx).all() and np.max(np.abs(w - r_w)) <= 1e-6


def test_single_cta_expert_gemm_wait_timeout_is_reported_and_the_context_stays_usable(monkeypatch):
    # 64 rows over 4 experts: below 256 rows per expert, the single-CTA kernel
    T, d, E, K, F = 32, 256, 4, 2, 192
    rng = np.random.default_rng(43)
    bf = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)
    x = bf(rng.normal(size=(T * K, d)))
    w13 = bf(rng.normal(size=(E, 2 * F, d)) / np.sqrt(d))
    w2 = bf(rng.normal(size=(E, d, F)) / np.sqrt(F))
    seg_off = np.array([0, 10, 30, 45, 64], dtype=np.int32)
    prob = api.make_problem(T, d, E, K, F, 0, 0.0, "bf16")
    ws = api.alloc_workspace(prob)
    R = api.max_rows(prob)
    x_rows = torch.zeros((R, d), dtype=torch.bfloat16)
    x_rows[:T * K] = x
    y_rows = torch.zeros((R, d), dtype=torch.bfloat16, device="cuda")

    def run():
        api.reset_device_status(ws)
        api.moe_expert_ffn(prob, api.FFN_ROUTED, dev(x_rows), R, dev(seg_off), dev(w13), dev(w2), y_rows, ws)
        t0 = time.monotonic()
        bits = api.read_device_status(ws)
        return bits, time.monotonic() - t0

    monkeypatch.setenv("MOE_B200_TEST_STALL_NS", STALL_NS)
    bits, waited = run()
    assert bits & DEV_WAIT_TIMEOUT, f"status {bits:#x}"
    assert waited < 10.0
    monkeypatch.delenv("MOE_B200_TEST_STALL_NS")
    bits, _ = run()
    assert bits == 0
    got = y_rows[:T * K].float().cpu().numpy()
    xs, W13, W2 = host_np(x), host_np(w13), host_np(w2)
    e_of = np.repeat(np.arange(E), np.diff(seg_off))
    x64 = (xs.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    want = np.stack([oracle.swiglu(x64[r], W13[e_of[r]], W2[e_of[r]]) for r in range(T * K)])
    assert rel_err(got, want) <= 2e-2
