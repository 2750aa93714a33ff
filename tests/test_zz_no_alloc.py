"""moe_dispatch_noalloc: the dispatch entry point for callers that cannot
allocate device memory for the library's scratch (a fixed device-memory
budget owned by their own pool, or no caching allocator, so that a cudaMalloc
per call would synchronise the device).  It must give exactly what
moe_dispatch gives with a workspace, call after call, although every call
reuses the library's one scratch array.  This file is collected last."""
import ctypes

import numpy as np
import pytest
import torch

from sparse_mixture_experts_04_b200 import _lib, api
from sparse_mixture_experts_04_b200.synth import MoeConfig, generate, given_logits

import oracle

CASES = [
    MoeConfig("na_mixtral", T=777, d_model=512, n_experts=8, top_k=2, d_ff=384, n_shared=0,
              capacity_factor=1.25, dtype="bf16", seed=31),
    MoeConfig("na_zen", T=1000, d_model=256, n_experts=128, top_k=8, d_ff=128, n_shared=0,
              capacity_factor=1.0, dtype="bf16", seed=32, bias_range=0.1),
    # above the fused scan+rank limit (ceil(T/256)^2 * E > 2^22): the separate
    # scan kernel writes the chunk bases into the second half of the array
    # (2 * 257 * 64 = 32896 of its 262144 words)
    MoeConfig("na_two_kernel_scan", T=65537, d_model=64, n_experts=64, top_k=4, d_ff=64, n_shared=0,
              capacity_factor=1.0, dtype="bf16", seed=33),
]


def _problem(cfg):
    return api.make_problem(cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff, cfg.n_shared,
                            cfg.capacity_factor, cfg.dtype)


def _outputs(cfg):
    R = max(api.max_rows(_problem(cfg)), 1)
    i32 = dict(dtype=torch.int32, device="cuda")
    return dict(counts=torch.empty(cfg.n_experts, **i32), kept=torch.empty(cfg.n_experts, **i32),
                seg_off=torch.empty(cfg.n_experts + 1, **i32),
                slot_of=torch.empty((cfg.T, cfg.top_k), **i32), perm=torch.full((R,), -9, **i32),
                x_perm=torch.zeros((R, cfg.d_model), dtype=torch.bfloat16, device="cuda"))


def _topk(cfg, shift):
    l = given_logits(cfg).astype(np.float64) + shift
    idx, _, _ = oracle.select(l, cfg.top_k)
    return torch.as_tensor(idx).cuda()


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_noalloc_dispatch_matches_workspace_dispatch_on_consecutive_calls(cfg):
    prob = _problem(cfg)
    x = generate(cfg, with_weights=False)["x"].cuda()
    ws = api.alloc_workspace(prob)
    rng = np.random.default_rng(cfg.seed)
    for call in range(2):   # the second call finds the first call's data in the shared array
        idx = _topk(cfg, rng.normal(size=cfg.n_experts) * (0.0 if call == 0 else 0.7))
        ref, got = _outputs(cfg), _outputs(cfg)
        api.moe_dispatch(prob, idx, x, ref["counts"], ref["kept"], ref["seg_off"], ref["slot_of"], ref["perm"],
                         ref["x_perm"], ws)
        api.moe_dispatch_noalloc(prob, idx, x, got["counts"], got["kept"], got["seg_off"], got["slot_of"],
                                 got["perm"], got["x_perm"])
        torch.cuda.synchronize()
        for k in ref:
            assert torch.equal(ref[k], got[k]), (call, k)


def test_noalloc_dispatch_rejects_problems_beyond_its_scratch():
    # 2 * ceil(T/256) * E words must fit in 262144: T = 200000, E = 256 needs 200704 * 2
    prob = api.make_problem(200000, 64, 256, 2, 64)
    fake = 4096
    rc = _lib.lib().moe_dispatch_noalloc(ctypes.byref(prob), fake, None, fake, fake, fake, fake, fake, None, None)
    assert rc == -2   # MOE_ERR_UNSUPPORTED, before anything touches the GPU
