"""The C-ABI library on the host (no GPU needed): it loads, exports every
symbol include/moe_b200.h declares, and its host-only functions and argument
checks behave as documented.  No call here reaches a kernel: every rejected
call returns before anything is enqueued."""
import ctypes
import os
import re

import pytest

import oracle
from sparse_mixture_experts_04_b200 import _lib, api, build
from sparse_mixture_experts_04_b200.synth import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(_lib.LIB_PATH):
        build.build()
    return _lib.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\**\s+\**(moe_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_layer_entry_points():
    names = declared_functions()
    for n in ("moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_layer_forward"):
        assert n in names
    assert sorted(_lib.EXPORTED) == names


def test_library_exports_every_declared_symbol(L):
    for n in declared_functions():
        assert hasattr(L, n), n
    assert L.moe_abi_version() == _lib.ABI_VERSION == 2


def test_status_strings(L):
    for code, name in _lib.STATUS_NAMES.items():
        assert L.moe_status_string(code).decode().startswith(name)


@pytest.mark.parametrize("name", list(CONFIGS))
def test_capacity_and_max_rows_match_definition(L, name):
    c = CONFIGS[name]
    prob = api.make_problem(c.T, c.d_model, c.n_experts, c.top_k, c.d_ff, c.n_shared, c.capacity_factor, c.dtype)
    cap = oracle.capacity(c.T, c.top_k, c.n_experts, c.capacity_factor)
    assert api.capacity(prob) == cap
    TK = c.T * c.top_k
    want_rows = TK if cap < 0 else min(TK, min(cap, c.T) * c.n_experts)
    assert api.max_rows(prob) == want_rows
    assert api.workspace_size(prob) > 0


@pytest.mark.parametrize("T,K,E,C", [(10, 1, 3, 1.0), (7, 2, 4, 0.5), (33, 3, 5, 1.1), (4, 4, 4, 2.0),
                                     (1000, 8, 128, 0.01), (1, 1, 1, 1.0)])
def test_capacity_edge_values(L, T, K, E, C):
    prob = api.make_problem(T, 64, E, K, 64, capacity_factor=C)
    assert api.capacity(prob) == oracle.capacity(T, K, E, C)


def _ret(fn, *args):
    return getattr(_lib.lib(), fn)(*args)


@pytest.mark.parametrize("field,value,code", [
    ("T", 0, -1), ("d_model", 12, -1), ("d_ff", 4, -1), ("n_experts", 0, -1), ("top_k", 0, -1),
    ("top_k", 9, -1), ("n_shared", -1, -1), ("dtype", 7, -1), ("flags", 0x20, -1), ("flags", 0x40, -1),
    ("n_experts", 300, -2), ("top_k", 33, -2)])
def test_invalid_problems_are_rejected(L, field, value, code):
    prob = api.make_problem(64, 64, 8, 2, 128)
    if field == "top_k" and value == 33:
        prob.n_experts = 64
    setattr(prob, field, value)
    n = ctypes.c_size_t(0)
    assert L.moe_workspace_size(ctypes.byref(prob), ctypes.byref(n)) == code
    assert L.moe_capacity(ctypes.byref(prob)) == -2


def test_entry_points_reject_bad_workspace_before_launching(L):
    prob = api.make_problem(64, 64, 8, 2, 128)
    P = ctypes.byref(prob)
    fake = 4096  # a non-null, 256-aligned address that is never dereferenced
    assert L.moe_route(P, fake, fake, None, None, fake, fake, fake, None, None, 0, None) == -5
    assert L.moe_route(P, fake, fake, None, None, fake, fake, fake, None, fake + 16, 1 << 30, None) == -5
    assert L.moe_route(P, fake, fake, None, None, fake, fake, fake, None, fake, 16, None) == -5
    assert L.moe_dispatch(P, fake, fake, fake, fake, fake, fake, fake, None, None, 0, None) == -5
    assert L.moe_expert_ffn(P, 0, fake, 8, fake, fake, fake, fake, None, 0, None) == -5
    assert L.moe_combine(P, fake, fake, fake, None, fake, None, 0, None) == -5
    w = _lib.MoeWeights(fake, None, None, fake, fake, None, None, None)
    assert L.moe_layer_forward(P, fake, ctypes.byref(w), fake, None, None, None, 0, None) == -5
    prob.flags = api.FLAG_EXPERT_CAPACITY
    assert L.moe_dispatch_capacity(P, fake, fake, fake, fake, fake, fake, fake, fake, None, None, 0, None) == -5


def test_entry_points_reject_bad_arguments_before_launching(L):
    prob = api.make_problem(64, 64, 8, 2, 128, n_shared=0)
    P = ctypes.byref(prob)
    n = ctypes.c_size_t(0)
    assert L.moe_workspace_size(P, ctypes.byref(n)) == 0
    ws, big = 1 << 20, n.value
    fake = 4096
    # required outputs missing
    assert L.moe_route(P, fake, fake, None, None, None, fake, fake, None, ws, big, None) == -1
    # misaligned x
    assert L.moe_route(P, fake + 4, fake, None, None, fake, fake, fake, None, ws, big, None) == -1
    # dispatch without slot_of
    assert L.moe_dispatch(P, fake, fake, fake, fake, fake, None, fake, None, ws, big, None) == -1
    # bad ffn mode; shared mode without shared experts; routed rows beyond max_rows
    assert L.moe_expert_ffn(P, 7, fake, 8, fake, fake, fake, fake, ws, big, None) == -1
    assert L.moe_expert_ffn(P, 1, fake, 8, None, fake, fake, fake, ws, big, None) == -1
    assert L.moe_expert_ffn(P, 0, fake, 64 * 2 + 1, fake, fake, fake, fake, ws, big, None) == -1
    # combine: y_shared given although n_shared == 0
    assert L.moe_combine(P, fake, fake, fake, fake, fake, ws, big, None) == -1
    # layer: logits-given mode needs routing.logits
    prob.flags = api.FLAG_LOGITS_GIVEN
    w = _lib.MoeWeights(None, None, None, fake, fake, None, None, None)
    assert L.moe_layer_forward(P, fake, ctypes.byref(w), fake, None, None, ws, big, None) == -1
    # layer: shared weights given although n_shared == 0
    prob.flags = 0
    w = _lib.MoeWeights(fake, None, None, fake, fake, fake, fake, None)
    assert L.moe_layer_forward(P, fake, ctypes.byref(w), fake, None, None, ws, big, None) == -1


def test_python_binding_raises_on_error(L):
    prob = api.make_problem(64, 64, 8, 2, 128)
    prob.top_k = 0
    with pytest.raises(api.MoeError):
        api.workspace_size(prob)


def test_expert_capacity_flag_sizes_for_all_pairs_and_checks_its_array(L):
    prob = api.make_problem(64, 64, 8, 2, 128, capacity_factor=0.5, flags=api.FLAG_EXPERT_CAPACITY)
    P = ctypes.byref(prob)
    assert api.capacity(prob) == 8          # the uniform capacity is still reported
    assert api.max_rows(prob) == 64 * 2     # but any expert may be given up to T rows
    n = ctypes.c_size_t(0)
    assert L.moe_workspace_size(P, ctypes.byref(n)) == 0
    ws, big, fake = 1 << 20, n.value, 4096
    # moe_dispatch has no capacity array: the flag needs moe_dispatch_capacity
    assert L.moe_dispatch(P, fake, fake, fake, fake, fake, fake, fake, None, ws, big, None) == -1
    assert L.moe_dispatch_capacity(P, fake, None, fake, fake, fake, fake, fake, fake, None, ws, big, None) == -1
    assert L.moe_dispatch_capacity(P, fake, fake + 4, fake, fake, fake, fake, fake, fake, None, ws, big, None) == -1
    # the layer reads the array from the weights
    w = _lib.MoeWeights(fake, None, None, fake, fake, None, None, None)
    assert L.moe_layer_forward(P, fake, ctypes.byref(w), fake, None, None, ws, big, None) == -1
    # moe_route cannot report drop figures for capacities it does not know
    prob.flags |= api.FLAG_EXTENDED_STATS
    assert L.moe_route(P, fake, fake, None, None, fake, fake, fake, fake, ws, big, None) == -1
    # moe_dispatch_capacity without the flag, and the no-workspace dispatch with it
    prob.flags = 0
    assert L.moe_dispatch_capacity(P, fake, fake, fake, fake, fake, fake, fake, fake, None, ws, big, None) == -1
    prob.flags = api.FLAG_EXPERT_CAPACITY
    assert L.moe_dispatch_noalloc(P, fake, fake, fake, fake, fake, fake, fake, None, None) == -1


@pytest.mark.parametrize("kw,why", [
    (dict(counts=None), "no counts"),
    (dict(sel_bias=None, expert_capacity=None), "nothing to update"),
    (dict(bias_rate=float("nan")), "non-finite rate"),
    (dict(bias_mode=2), "unknown mode"),
    (dict(count_hist=None), "capacity without history"),
    (dict(hist_len=0), "empty history"),
    (dict(step=-1), "negative step"),
    (dict(c_base=0.0), "no base capacity"),
    (dict(gamma=float("inf")), "non-finite gamma"),
    (dict(sel_bias=4096 + 8), "misaligned bias"),
])
def test_balance_update_rejects_bad_arguments(L, kw, why):
    prob = api.make_problem(64, 64, 8, 2, 128, capacity_factor=1.0)
    fake = 4096
    a = dict(counts=fake, sel_bias=fake, bias_rate=0.01, bias_mode=0, count_hist=fake, hist_len=4, step=0,
             c_base=1.0, gamma=0.5, expert_capacity=fake)
    a.update(kw)
    rc = L.moe_balance_update(ctypes.byref(prob), a["counts"], a["sel_bias"], a["bias_rate"], a["bias_mode"],
                              a["count_hist"], a["hist_len"], a["step"], a["c_base"], a["gamma"],
                              a["expert_capacity"], None)
    assert rc == -1, why


def test_backward_rejects_bad_arguments_before_launching(L):
    fake = 4096
    prob = api.make_problem(64, 64, 8, 2, 128, capacity_factor=1.0)
    P = ctypes.byref(prob)
    n = ctypes.c_size_t(0)
    assert L.moe_workspace_size(P, ctypes.byref(n)) == 0
    fwd = n.value
    assert L.moe_backward_workspace_size(P, ctypes.byref(n)) == 0 and n.value > 0
    bwd = n.value
    w = _lib.MoeWeights(fake, None, None, fake, fake, None, None, None)
    good = _lib.MoeGrads(fake, fake, fake, None, None, fake, None, None)

    def call(prob_=prob, x=fake, g=good, fws=fake, fbytes=fwd, dy=fake, ws=1 << 20, wbytes=bwd, d_loss=1.0):
        return L.moe_layer_backward(ctypes.byref(prob_), x, ctypes.byref(w), None, fws, fbytes, dy, d_loss, 0.0,
                                    ctypes.byref(g), ws, wbytes, None)

    assert call(dy=None) == -1
    assert call(x=fake + 4) == -1
    assert call(d_loss=float("nan")) == -1
    assert call(g=_lib.MoeGrads(fake, None, fake, None, None, None, None, None)) == -1   # dw13 required
    assert call(g=_lib.MoeGrads(fake, fake, fake, fake, fake, None, None, None)) == -1   # shared grads, no shared
    assert call(fbytes=fwd - 1) == -5
    assert call(wbytes=bwd - 1) == -5
    assert call(ws=(1 << 20) + 16) == -5
    f32 = api.make_problem(64, 64, 8, 2, 128, dtype="f32")
    assert call(prob_=f32) == -2
    given = api.make_problem(64, 64, 8, 2, 128, flags=api.FLAG_LOGITS_GIVEN)
    assert call(prob_=given) == -1   # dw_gate requested although the logits are given


def test_peer_exchange_entry_points_reject_bad_arguments_before_launching(L):
    """moe_ep_peer_plan / moe_ep_scatter / moe_ep_combine and the IPC calls
    refuse bad arguments on the host, before any launch or CUDA call."""
    prob = api.make_problem(64, 64, 8, 2, 128, n_shared=0)
    P = ctypes.byref(prob)
    fake = 4096
    # plan: rank out of range, E not divisible by G, E above 256, NULL outputs
    assert L.moe_ep_peer_plan(2, 2, 8, fake, fake, fake, None) == -1
    assert L.moe_ep_peer_plan(3, 0, 8, fake, fake, fake, None) == -1
    assert L.moe_ep_peer_plan(1, 0, 512, fake, fake, fake, None) == -1
    assert L.moe_ep_peer_plan(2, 0, 8, fake, None, fake, None) == -1
    # scatter: G does not divide E; misaligned x; NULL table
    assert L.moe_ep_scatter(P, 3, fake, fake, fake, fake, fake, None) == -1
    assert L.moe_ep_scatter(P, 2, fake + 4, fake, fake, fake, fake, None) == -1
    assert L.moe_ep_scatter(P, 2, fake, fake, fake, None, fake, None) == -1
    # combine: y_shared given although n_shared == 0; misaligned y; G does not divide E
    assert L.moe_ep_combine(P, 2, fake, fake, fake, fake, fake, fake, fake, None) == -1
    assert L.moe_ep_combine(P, 2, fake, fake, fake, fake, fake, None, fake + 8, None) == -1
    assert L.moe_ep_combine(P, 3, fake, fake, fake, fake, fake, None, fake, None) == -1
    # IPC: NULL arguments, zero bytes
    p = ctypes.c_void_p()
    assert L.moe_ipc_malloc(0, ctypes.byref(p)) == -1
    assert L.moe_ipc_handle(None, fake) == -1
    assert L.moe_ipc_open(None, ctypes.byref(p)) == -1
    assert L.moe_ipc_close(None) == -1 and L.moe_ipc_free(None) == -1
