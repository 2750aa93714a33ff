"""B200 (sm_100a) sparse Mixture-of-Experts FFN forward.

The layer runs in libmoe_b200.so (hand-written CUDA kernels behind a C ABI,
include/moe_b200.h); this package is its Python binding.  The library is
loaded on first use and its absence is an error.

Modules:
  api    -- the C entry points with torch tensors (moe_route, moe_dispatch,
            moe_expert_ffn, moe_combine, moe_layer_forward, ...)
  layer  -- MoeLayer: weights + workspace held on the device, forward()
  ep     -- expert-parallel forward: experts split over ranks, rows exchanged
            with torch.distributed point-to-point (moe_ep_plan plans it)
  synth  -- seeded synthetic inputs of the five workloads
  build  -- nvcc build of the library
"""
from .api import *  # noqa: F401,F403
from .api import __all__ as _api_all
from .layer import MoeLayer  # noqa: F401

__all__ = list(_api_all) + ["MoeLayer"]
