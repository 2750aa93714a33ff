"""The layer forward captured into a CUDA graph (MoeLayer.capture /
forward_graphed): every replay equals the eager forward of the same input,
bit for bit (the kernels are deterministic), routing and statistics included,
for inputs that change between replays."""
import pytest
import torch

from helpers import dev, generate
from sparse_mixture_experts_04_b200 import MoeLayer, api
from sparse_mixture_experts_04_b200.synth import CONFIGS, MoeConfig, extra_activations

pytestmark = pytest.mark.gpu

CFGS = {
    "small_bf16": MoeConfig("graph_small", T=300, d_model=256, n_experts=8, top_k=2, d_ff=384, n_shared=1,
                            capacity_factor=1.0, dtype="bf16", seed=31, x_std=1.0),
    "pairs_bf16": MoeConfig("graph_pairs", T=1536, d_model=512, n_experts=8, top_k=2, d_ff=1024, n_shared=0,
                            capacity_factor=1.25, dtype="bf16", seed=32, x_std=1.0),
    "tiny_fp32": CONFIGS["tiny_fp32"],
}


@pytest.mark.parametrize("name", list(CFGS))
def test_graph_replays_equal_eager_forwards(name):
    cfg = CFGS[name]
    inp = generate(cfg)
    layer = MoeLayer.from_inputs(inp, flags=api.FLAG_EXTENDED_STATS)
    xs = [dev(x) for x in [inp["x"]] + extra_activations(cfg, 3)]
    want = []
    for x in xs:
        y = layer.forward(x)
        want.append((y.clone(), layer.stats.clone(), layer.routing["topk_idx"].clone(),
                     layer.routing["slot_of"].clone()))
    layer.capture()
    for i in (2, 0, 3, 1, 1):
        y = layer.forward_graphed(xs[i])
        torch.cuda.synchronize()
        assert api.read_device_status(layer.ws) == 0
        y_w, st_w, idx_w, slot_w = want[i]
        assert torch.equal(y, y_w)
        assert torch.equal(layer.stats, st_w)
        assert torch.equal(layer.routing["topk_idx"], idx_w)
        assert torch.equal(layer.routing["slot_of"], slot_w)


def test_forward_graphed_needs_capture():
    cfg = CFGS["small_bf16"]
    layer = MoeLayer.from_inputs(generate(cfg))
    with pytest.raises(RuntimeError):
        layer.forward_graphed()
