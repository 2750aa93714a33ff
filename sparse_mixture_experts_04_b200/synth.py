"""Seeded synthetic inputs for the sparse-MoE FFN layer.

This module is shared by the tests, the benchmark and the smoke check: it is
the one thing both the CUDA path and the float64 oracle are fed from.  It
holds none of the layer's arithmetic -- it only draws random tensors with the
shapes and distributions of the five workloads and rounds them to the storage
type.  (The Zipf logit offsets of the skewed workload are an input
distribution, not part of the method.)

Recipe (every tensor has its own PCG64 stream, keyed by (seed, tensor id) --
and per expert matrix by (seed, tensor id, expert) -- so a tensor does not
change when another tensor's size changes):
  x          N(0, x_std^2)                              [T, d]
  w_gate     N(0, 1/d)                                   [E, d]
  w13        N(0, 1/d)   rows 0..F-1 gate, F..2F-1 up    [E, 2F, d]
  w2         N(0, 1/F)                                   [E, d, F]
  w13_shared / w2_shared  as w13 / w2                    [N_s, 2F, d] / [N_s, d, F]
  sel_bias   U(-r, r), float32 (selection-only bias)     [E]
  logit_offset  -s * ln(rank_e), rank = seeded permutation of 1..E, float32;
             exp(offset) is then a Zipf(s) popularity prior over experts  [E]
  logits     N(0, sigma^2) (+ logit_offset), float32, for routing tests that
             feed the same logits to both sides; sigma is the standard
             deviation of x . w_gate under the recipe above   [T, E]
BF16 tensors are float32 draws rounded to nearest-even BF16 (via torch).
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os
from dataclasses import dataclass

import numpy as np
import torch

# tensor ids of the per-tensor random streams
_X, _WG, _W13, _W2, _W13S, _W2S, _BIAS, _OFF, _LOGITS = range(1, 10)


@dataclass(frozen=True)
class MoeConfig:
    name: str
    T: int
    d_model: int
    n_experts: int
    top_k: int
    d_ff: int
    n_shared: int
    capacity_factor: float      # <= 0: no capacity limit
    dtype: str                  # "bf16" or "f32"
    seed: int
    x_std: float = 1.0
    bias_range: float = 0.0     # > 0: per-expert selection bias U(-r, r)
    zipf_s: float = 0.0         # > 0: Zipf(s) logit offsets
    alpha: float = 0.01
    description: str = ""

    def replace(self, **kw) -> "MoeConfig":
        return dataclasses.replace(self, **kw)

    @property
    def logit_std(self) -> float:
        # std of sum_j x_j w_j with x ~ N(0, x_std^2), w ~ N(0, 1/d)
        return self.x_std


CONFIGS = {
    "tiny_fp32": MoeConfig(
        "tiny_fp32", T=64, d_model=64, n_experts=8, top_k=2, d_ff=128, n_shared=0,
        capacity_factor=0.0, dtype="f32", seed=0, x_std=1.0 / math.sqrt(64),
        description="Tiny MoE layer, FP32: T=64, d=64, E=8, top-2, F=128, no shared, no capacity limit"),
    "mixtral": MoeConfig(
        "mixtral", T=4096, d_model=4096, n_experts=8, top_k=2, d_ff=14336, n_shared=0,
        capacity_factor=1.25, dtype="bf16", seed=1,
        description="Mixtral-shaped layer, BF16: T=4096, d=4096, E=8, top-2, F=14336, C=1.25"),
    "zen_fine": MoeConfig(
        "zen_fine", T=8192, d_model=2048, n_experts=128, top_k=8, d_ff=1024, n_shared=4,
        capacity_factor=1.0, dtype="bf16", seed=2, bias_range=0.1,
        description="Fine-grained layer, BF16: T=8192, d=2048, E=128 top-8 + 4 shared, F=1024, C=1.0, "
                    "selection bias U(-0.1, 0.1)"),
    "skewed": MoeConfig(
        "skewed", T=16384, d_model=2048, n_experts=64, top_k=4, d_ff=1408, n_shared=0,
        capacity_factor=1.0, dtype="bf16", seed=3, zipf_s=1.2,
        description="Skewed-load layer, BF16: T=16384, d=2048, E=64, top-4, F=1408, C=1.0, "
                    "Zipf(1.2) logit offsets"),
    "decode": MoeConfig(
        "decode", T=32, d_model=4096, n_experts=128, top_k=8, d_ff=1536, n_shared=1,
        capacity_factor=0.0, dtype="bf16", seed=4,
        description="Decode-shaped layer, BF16: T=32, d=4096, E=128 top-8 + 1 shared, F=1536, no limit"),
}


def _rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(tensor_id)])))


def _normal(rng: np.random.Generator, shape, std: float, dtype: str) -> torch.Tensor:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    a *= np.float32(std)
    t = torch.from_numpy(a)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _normal_stack(seed, tensor_id, n, shape, std, dtype) -> torch.Tensor:
    """n independent matrices, matrix i from stream (seed, tensor_id, i); drawn
    on a few threads (the generator's fill releases the GIL)."""
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = torch.empty((n,) + tuple(shape), dtype=tdt)

    def one(i):
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(tensor_id), i])))
        out[i] = _normal(rng, shape, std, dtype)

    workers = max(1, min(n, os.cpu_count() or 1, 16))
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        list(ex.map(one, range(n)))
    return out


def zipf_offsets(cfg: MoeConfig) -> np.ndarray:
    rank = _rng(cfg.seed, _OFF).permutation(cfg.n_experts).astype(np.float64) + 1.0
    return (-cfg.zipf_s * np.log(rank)).astype(np.float32)


def generate(cfg: MoeConfig, with_weights: bool = True) -> dict:
    """All layer inputs as CPU tensors (BF16 or FP32) plus float32 numpy extras."""
    T, d, E, F, Ns = cfg.T, cfg.d_model, cfg.n_experts, cfg.d_ff, cfg.n_shared
    out = {"cfg": cfg}
    out["x"] = _normal(_rng(cfg.seed, _X), (T, d), cfg.x_std, cfg.dtype)
    out["w_gate"] = _normal(_rng(cfg.seed, _WG), (E, d), 1.0 / math.sqrt(d), cfg.dtype)
    if with_weights:
        out["w13"] = _normal_stack(cfg.seed, _W13, E, (2 * F, d), 1.0 / math.sqrt(d), cfg.dtype)
        out["w2"] = _normal_stack(cfg.seed, _W2, E, (d, F), 1.0 / math.sqrt(F), cfg.dtype)
        if Ns > 0:
            out["w13_shared"] = _normal_stack(cfg.seed, _W13S, Ns, (2 * F, d), 1.0 / math.sqrt(d), cfg.dtype)
            out["w2_shared"] = _normal_stack(cfg.seed, _W2S, Ns, (d, F), 1.0 / math.sqrt(F), cfg.dtype)
        else:
            out["w13_shared"] = None
            out["w2_shared"] = None
    out["sel_bias"] = (_rng(cfg.seed, _BIAS).uniform(-cfg.bias_range, cfg.bias_range, size=E).astype(np.float32)
                       if cfg.bias_range > 0 else None)
    out["logit_offset"] = zipf_offsets(cfg) if cfg.zipf_s > 0 else None
    return out


def extra_activations(cfg: MoeConfig, n: int) -> list:
    """n further activation batches x [T, d] with the recipe of x, from streams
    (seed, 100 + i); used to rotate inputs between timed steps."""
    return [_normal(_rng(cfg.seed, 100 + i), (cfg.T, cfg.d_model), cfg.x_std, cfg.dtype) for i in range(n)]


def given_logits(cfg: MoeConfig, T: int | None = None) -> np.ndarray:
    """float32 router logits with the workload's statistics (see module doc)."""
    T = cfg.T if T is None else T
    l = _rng(cfg.seed, _LOGITS).standard_normal(size=(T, cfg.n_experts), dtype=np.float32)
    l *= np.float32(cfg.logit_std)
    if cfg.zipf_s > 0:
        l += zipf_offsets(cfg)[None, :]
    return l


def exact_router_inputs(T: int, d: int, E: int, seed: int) -> dict:
    """Router inputs whose gate logits are exact in float32: x entries k/8 with
    k in [-4, 4], w_gate integers in [-3, 3], offsets multiples of 1/8 in
    [-1, 1].  Every product is a multiple of 1/8 of magnitude <= 1.5, so every
    partial sum (d <= 4096) is a multiple of 1/8 below 2^13 in magnitude and
    exact in float32: any summation order gives the same float32 (and float64)
    value, and many logits tie exactly."""
    assert d <= 4096
    rng = np.random.default_rng(seed)
    x = torch.from_numpy(rng.integers(-4, 5, size=(T, d)).astype(np.float32) / 8).to(torch.bfloat16)
    w = torch.from_numpy(rng.integers(-3, 4, size=(E, d)).astype(np.float32)).to(torch.bfloat16)
    off = (rng.integers(-8, 9, size=E) / 8).astype(np.float32)
    return {"x": x, "w_gate": w, "logit_offset": off}


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw BF16 bits of a CPU bfloat16 tensor, as uint16 numpy (for the oracle)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
