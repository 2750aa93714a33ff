"""GPU parity of the layer backward (moe_layer_backward) against the float64
oracle's backward (itself pinned by finite differences of the forward).

Inputs: x and the gate weights from exact_router_inputs, so the GPU's logits
equal the oracle's exactly and both sides route identically (checked); expert
weights and dy seeded normal, BF16.  Bar: max|g - g_ref| / max|g_ref| per
gradient tensor within BWD_TOL.  The backward rounds three chained
intermediates to BF16 (do rows, dg/du, dx rows; and the logit gradient fed to
the gate GEMMs), each a relative error of at most 2^-9, so its error is a few
times the forward's; 3e-2 leaves room for that."""
import numpy as np
import pytest
import torch

import oracle
from helpers import dev, host_np, rel_err
from sparse_mixture_experts_04_b200 import MoeLayer, api
from sparse_mixture_experts_04_b200.synth import exact_router_inputs

pytestmark = pytest.mark.gpu
BWD_TOL = 3e-2

CASES = {  # T, d, E, K, F, Ns, C, bias
    "mixtral_like": (300, 256, 8, 2, 384, 0, 1.25, None),
    "drops_shared": (257, 128, 16, 4, 200, 2, 0.6, "prob"),
    "fine_e64": (500, 192, 64, 6, 136, 1, 1.0, "logit"),
    "e7_ragged": (129, 264, 7, 3, 72, 1, 0.9, None),
    "single_expert": (64, 64, 1, 1, 64, 0, 0.0, None),
    # groups of ~300 rows and d, F multiples of 64: the CTA-pair backward GEMMs
    # (dgrad tiles of 256 rows, wgrad k-blocks of 128 rows with a tail)
    "pairs_shared": (600, 256, 4, 2, 320, 1, 1.25, None),
}


def _inputs(name):
    T, d, E, K, F, Ns, C, bias = CASES[name]
    rng = np.random.default_rng(len(name) * 31 + T)
    inp = exact_router_inputs(T, d, E, seed=T + E)
    bf = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)
    inp["w13"] = bf(rng.normal(size=(E, 2 * F, d)) / np.sqrt(d))
    inp["w2"] = bf(rng.normal(size=(E, d, F)) / np.sqrt(F))
    inp["w13_shared"] = bf(rng.normal(size=(Ns, 2 * F, d)) / np.sqrt(d)) if Ns else None
    inp["w2_shared"] = bf(rng.normal(size=(Ns, d, F)) / np.sqrt(F)) if Ns else None
    inp["sel_bias"] = None if bias is None else rng.uniform(-0.02, 0.02, size=E).astype(np.float32)
    dy = bf(rng.normal(size=(T, d)))
    flags = api.FLAG_BIAS_LOGIT if bias == "logit" else 0
    prob = api.make_problem(T, d, E, K, F, Ns, C, "bf16", flags, 0.01)
    return prob, inp, dy


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("d_loss,d_zloss,save_gu", [(1.0, 0.0, False), (0.5, 2.0, False), (1.0, 0.5, True)])
def test_layer_backward_matches_oracle(name, d_loss, d_zloss, save_gu):
    """save_gu: the forward keeps the gate/up projections (MOE_FLAG_SAVE_GU)
    instead of the backward recomputing them."""
    prob, inp, dy = _inputs(name)
    if save_gu:
        prob.flags |= api.FLAG_SAVE_GU
    T, d, E, K, F, Ns = prob.T, prob.d_model, prob.n_experts, prob.top_k, prob.d_ff, prob.n_shared
    w = {k: dev(inp.get(k)) for k in ("w_gate", "w13", "w2", "w13_shared", "w2_shared", "sel_bias", "logit_offset")}
    layer = MoeLayer(prob, w)
    x = dev(inp["x"])
    layer.forward(x)
    g = layer.backward(x, dev(dy), d_loss, d_zloss)
    torch.cuda.synchronize()
    assert api.read_device_status(layer.ws) == 0

    l64 = oracle.gate_logits(host_np(inp["x"]), host_np(inp["w_gate"]), inp["logit_offset"])
    assert (layer.routing["logits"].cpu().numpy().astype(np.float64) == l64).all()
    mode = oracle.BIAS_LOGIT if prob.flags & api.FLAG_BIAS_LOGIT else oracle.BIAS_PROB
    idx, wgt, p = oracle.select(l64, K, bias=inp["sel_bias"], bias_mode=mode)
    disp = oracle.dispatch(idx, E, oracle.capacity(T, K, E, prob.capacity_factor))
    assert (layer.routing["topk_idx"].cpu().numpy() == idx).all()
    assert (layer.routing["slot_of"].cpu().numpy() == disp["slot_of"]).all()
    ref = oracle.layer_backward(host_np(inp["x"]), host_np(inp["w_gate"]), host_np(inp["w13"]), host_np(inp["w2"]),
                                l64, idx, wgt, disp["slot_of"], disp["counts"], 0.01,
                                dy.float().numpy().astype(np.float64), d_loss, d_zloss,
                                host_np(inp["w13_shared"]) if Ns else None, host_np(inp["w2_shared"]) if Ns else None)
    checks = [("dx", g["dx"].float()), ("dw13", g["dw13"]), ("dw2", g["dw2"]), ("dwg", g["dw_gate"]),
              ("doff", g["d_offset"]), ("dlogits", g["d_logits"])]
    if Ns:
        checks += [("dw13_shared", g["dw13_shared"]), ("dw2_shared", g["dw2_shared"])]
    for key, got in checks:
        err = rel_err(got.cpu().numpy(), ref[key])
        assert err <= BWD_TOL, f"{key}: {err:.3e}"
    # experts without kept rows get exactly zero
    for e in range(E):
        if disp["kept"][e] == 0:
            assert not g["dw13"][e].any() and not g["dw2"][e].any()


@pytest.mark.parametrize("name", ["pairs_shared", "mixtral_like"])
def test_single_cta_and_pair_backward_gemms_agree(name, monkeypatch):
    """The same backward with the CTA-pair GEMMs (the default where the shapes
    allow) and with the single-CTA ones (MOE_B200_GRAD_PAIR=0): both within the
    oracle bar above; here they must agree to BF16 rounding of the stored
    intermediates (dg/du, dx rows) and FP32 summation order (weights)."""
    prob, inp, dy = _inputs(name)
    w = {k: dev(inp.get(k)) for k in ("w_gate", "w13", "w2", "w13_shared", "w2_shared", "sel_bias", "logit_offset")}
    x = dev(inp["x"])
    out = []
    for env in ("1", "0"):
        monkeypatch.setenv("MOE_B200_GRAD_PAIR", env)
        layer = MoeLayer(prob, w)
        layer.forward(x)
        out.append({k: v.float().clone() for k, v in layer.backward(x, dev(dy), 1.0, 0.5).items()})
        assert api.read_device_status(layer.ws) == 0
    for k in out[0]:
        assert rel_err(out[0][k].cpu().numpy(), out[1][k].cpu().numpy().astype(np.float64)) <= 1e-2, k


def test_layer_backward_is_deterministic():
    prob, inp, dy = _inputs("drops_shared")
    w = {k: dev(inp.get(k)) for k in ("w_gate", "w13", "w2", "w13_shared", "w2_shared", "sel_bias", "logit_offset")}
    layer = MoeLayer(prob, w)
    x = dev(inp["x"])
    layer.forward(x)
    g1 = {k: v.clone() for k, v in layer.backward(x, dev(dy), 1.0, 1.0).items()}
    g2 = layer.backward(x, dev(dy), 1.0, 1.0)
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


def test_saved_projections_give_the_same_gradients_as_recomputed():
    prob, inp, dy = _inputs("drops_shared")
    w = {k: dev(inp.get(k)) for k in ("w_gate", "w13", "w2", "w13_shared", "w2_shared", "sel_bias", "logit_offset")}
    x = dev(inp["x"])
    grads = []
    for flags in (0, api.FLAG_SAVE_GU):
        p2 = api.make_problem(prob.T, prob.d_model, prob.n_experts, prob.top_k, prob.d_ff, prob.n_shared,
                              prob.capacity_factor, "bf16", prob.flags | flags, prob.alpha)
        layer = MoeLayer(p2, w)
        layer.forward(x)
        grads.append({k: v.clone() for k, v in layer.backward(x, dev(dy), 1.0, 1.0).items()})
    for k in grads[0]:
        assert torch.equal(grads[0][k], grads[1][k]), k
