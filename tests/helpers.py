"""Shared test helpers: oracle references for a synthetic workload and small
device-transfer utilities.  Expected values come only from the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_mixture_experts_04_b200 import api
from sparse_mixture_experts_04_b200.synth import MoeConfig, bf16_bits, generate, given_logits

BF16_TOL = 2e-2   # max |y - y_ref| / max |y_ref|, BF16 layer outputs
F32_TOL = 1e-4    # same, FP32 layer outputs


def bias_mode(flags: int) -> int:
    return oracle.BIAS_LOGIT if flags & api.FLAG_BIAS_LOGIT else oracle.BIAS_PROB


def host_np(t):
    """CPU tensor -> numpy input for the oracle (BF16 as raw uint16 bits)."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t
    if t.dtype == torch.bfloat16:
        return bf16_bits(t)
    return t.contiguous().numpy()


def oracle_routing(cfg: MoeConfig, logits64: np.ndarray, sel_bias, flags: int = 0) -> dict:
    idx, w, p = oracle.select(logits64, cfg.top_k, bias=sel_bias, bias_mode=bias_mode(flags))
    cap = oracle.capacity(cfg.T, cfg.top_k, cfg.n_experts, cfg.capacity_factor)
    disp = oracle.dispatch(idx, cfg.n_experts, cap)
    f, P, loss = oracle.balance(disp["counts"], p, cfg.top_k, cfg.alpha)
    return dict(idx=idx, w=w, p=p, cap=cap, f=f, P=P, loss=loss, **disp)


def oracle_layer(inp: dict, route: dict, rows=None) -> np.ndarray:
    return oracle.layer_rows(host_np(inp["x"]), host_np(inp["w13"]), host_np(inp["w2"]), route["idx"], route["w"],
                             route["slot_of"], rows=rows, w13_shared=host_np(inp.get("w13_shared")),
                             w2_shared=host_np(inp.get("w2_shared")))


def rel_err(got: np.ndarray, want: np.ndarray) -> float:
    denom = float(np.max(np.abs(want)))
    if denom == 0.0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got.astype(np.float64) - want))) / denom


def tol(cfg: MoeConfig) -> float:
    return BF16_TOL if cfg.dtype == "bf16" else F32_TOL


def dev(t, device="cuda"):
    if t is None:
        return None
    return torch.as_tensor(t).to(device).contiguous()


def problem(cfg: MoeConfig, flags: int = 0) -> api.MoeProblem:
    return api.make_problem(cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff, cfg.n_shared,
                            cfg.capacity_factor, cfg.dtype, flags, cfg.alpha)


def sample_rows(T: int, n: int, seed: int, extra=()) -> np.ndarray:
    """Deterministic sample of token rows: edges, chunk borders, random."""
    rng = np.random.default_rng(seed)
    fixed = {0, T - 1, min(T - 1, 255), min(T - 1, 256), min(T - 1, 127), T // 2, *extra}
    rest = rng.choice(T, size=min(T, n), replace=False)
    return np.array(sorted(set(int(r) for r in fixed if 0 <= r < T) | set(int(r) for r in rest)), dtype=np.int64)


__all__ = ["oracle_routing", "oracle_layer", "rel_err", "tol", "dev", "problem", "sample_rows", "host_np",
           "generate", "given_logits", "BF16_TOL", "F32_TOL"]
