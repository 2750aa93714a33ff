"""Host-side arithmetic of bench.py: the roofline's bound and byte counts."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from sparse_mixture_experts_04_b200.synth import CONFIGS  # noqa: E402

PEAKS = {"hbm_gbs": 6540.8, "bf16_tflops": 1641.2, "bf16_tflops_sustained": 1380.6}


def test_up_gemm_bytes_counts_touched_experts_rows_and_h():
    cfg = CONFIGS["mixtral"]
    kept = [1024] * 7 + [0]
    d, F = cfg.d_model, cfg.d_ff
    want = 2 * (7 * 2 * F * d + 7 * 1024 * d + 7 * 1024 * F)
    assert bench.up_gemm_bytes(cfg, kept) == want


def test_roofline_is_tensor_bound_for_large_groups():
    cfg = CONFIGS["mixtral"]
    kept = [1024] * 8
    flops = bench.algorithmic_flops(cfg, sum(kept))["up"]
    nbytes = bench.up_gemm_bytes(cfg, kept)
    # a timed region under a second: the burst peak, the sustained one beside it
    r = bench.roofline(cfg, flops, nbytes, 1.5, PEAKS, "measured", None, 0.12)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(flops / 1.5e-3 / 1e12)
    assert r["peak"] == PEAKS["bf16_tflops"] and "burst" in r["peak_source"]
    assert r["frac"] == pytest.approx(r["achieved"] / PEAKS["bf16_tflops"])
    assert r["frac_of_sustained"] == pytest.approx(r["achieved"] / PEAKS["bf16_tflops_sustained"])
    # a timed region of seconds runs under the power limit: the sustained peak
    r = bench.roofline(cfg, flops, nbytes, 1.5, PEAKS, "measured", None, 3.0)
    assert r["peak"] == PEAKS["bf16_tflops_sustained"] and "sustained" in r["peak_source"]
    assert r["frac_of_burst"] == pytest.approx(r["achieved"] / PEAKS["bf16_tflops"])
    burst_only = {k: v for k, v in PEAKS.items() if k != "bf16_tflops_sustained"}
    r = bench.roofline(cfg, flops, nbytes, 1.5, burst_only, "fallback", None, 3.0)
    assert r["peak"] == PEAKS["bf16_tflops"] and "burst" in r["peak_source"]


def test_roofline_is_hbm_bound_when_weights_dominate():
    cfg = CONFIGS["decode"]
    kept = [2] * cfg.n_experts          # a few rows per expert: weight streaming
    flops = bench.algorithmic_flops(cfg, sum(kept))["up"]
    nbytes = bench.up_gemm_bytes(cfg, kept)
    r = bench.roofline(cfg, flops, nbytes, 0.5, PEAKS, "fallback", None, 0.04)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(nbytes / 0.5e-3 / 1e9)
    assert r["peak"] == PEAKS["hbm_gbs"] and "fallback" in r["peak_source"]


def test_router_and_combine_bytes_at_the_mixtral_shape():
    """x (33.6 MB) dominates the router; the combine reads the 8192 kept rows
    (67 MB) and writes y (33.5 MB): about 101 MB."""
    cfg = CONFIGS["mixtral"]
    T, d, E, K = cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k
    assert bench.router_bytes(cfg) == 2 * T * d + 2 * E * d + 4 * T * E + 8 * T * K
    assert 33.5e6 < bench.router_bytes(cfg) < 34.0e6
    kept = T * K
    assert bench.combine_bytes(cfg, kept) == 2 * kept * d + 2 * T * d + 8 * T * K
    assert 100e6 < bench.combine_bytes(cfg, kept) < 101.5e6
    # a shared expert adds its output rows to the combine's reads
    z = CONFIGS["zen_fine"]
    assert bench.combine_bytes(z, 0) == 2 * z.T * z.d_model * 2 + 8 * z.T * z.top_k


@pytest.mark.parametrize("name,want", [("zen_fine", True), ("mixtral", False), ("skewed", False), ("decode", True),
                                       ("tiny_fp32", False)])
def test_shared_mixed_follows_the_library_rule(name, want, monkeypatch):
    """The shared experts share the routed launches only with BF16, shared
    experts and the same tile shape for both (CTA pairs: >= 256 expected rows
    per routed expert after the capacity and T >= 256; single CTAs: both
    below); MOE_B200_MIX_SHARED=0 turns it off."""
    from sparse_mixture_experts_04_b200 import api
    cfg = CONFIGS[name]
    prob = api.make_problem(cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff, cfg.n_shared,
                            cfg.capacity_factor, cfg.dtype)
    assert bench.shared_mixed(cfg, prob) is want
    monkeypatch.setenv("MOE_B200_MIX_SHARED", "0")
    assert bench.shared_mixed(cfg, prob) is False


def test_shared_up_bytes_counts_weights_x_and_h():
    cfg = CONFIGS["zen_fine"]
    d, F, Ns, T = cfg.d_model, cfg.d_ff, cfg.n_shared, cfg.T
    assert bench.shared_up_bytes(cfg) == 2 * (Ns * 2 * F * d + T * d + T * Ns * F)


def test_stage_spans_from_device_clocks():
    """Each stage's pair holds (~earliest start, latest end); dispatch+gather
    runs from the dispatch kernels' start to the gather's end; stages left at
    zero (not run, or not stamped) are absent."""
    from sparse_mixture_experts_04_b200 import _lib
    n = _lib.NUM_CLOCKS
    names = _lib.CLOCK_NAMES
    row = [0] * (2 * n)
    mask = (1 << 64) - 1

    def put(name, start_ns, end_ns):
        i = names.index(name)
        c = (~start_ns) & mask
        row[2 * i] = c - (1 << 64) if c >= 1 << 63 else c   # int64 as torch returns it
        row[2 * i + 1] = end_ns

    put("route", 1_000, 9_000)
    put("dispatch", 10_000, 14_000)
    put("gather", 14_500, 35_000)
    put("combine", 40_000, 60_000)
    spans = bench.stage_spans([row, row])
    assert spans["route"] == pytest.approx(8.0)
    assert spans["dispatch+gather"] == pytest.approx(25.0)
    assert spans["gather"] == pytest.approx(20.5)
    assert spans["combine"] == pytest.approx(20.0)
    assert "up" not in spans and "shared" not in spans
