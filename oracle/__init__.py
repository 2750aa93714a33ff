"""Float64 CPU oracle for the sparse-MoE FFN forward -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library in
``sparse_mixture_experts_04_b200``) never imports, links or calls it, and the
two share no code.  The arithmetic lives in ``moe_oracle.c`` (plain loops,
float64); this module only marshals numpy arrays into it.  It runs on one
thread unless ``set_threads(n)`` with n > 1 switches to the same source built
with OpenMP (outer loops of the gate logits and layer rows split over
threads, every output still summed in the same order: the same bits).

Every function here names the passage it follows (page title and section /
equation); see the header of ``moe_oracle.c`` for the source list.

Parity pins (what ties each function to something other than itself) are in
``tests/test_oracle.py``:
  gate_logits    hand-built one-hot weights, exact integer dot products
  softmax        closed form for two experts, sums to one, shift invariance
  select         brute-force full sort on tiny inputs; tie rule; renormalisation
  capacity       exact integer cases printed in the configs' arithmetic
  dispatch       brute force per-expert queues; bijection and order invariants
  dispatch_caps  brute force per-expert queues with a different capacity per expert
  bias_update    hand-worked loads: overloaded down, underloaded up, balanced unchanged;
                 proportional steps sum to zero; a fixed routing drives the biases apart
  adaptive_capacity  hand-worked C_e / cap_e; gamma = 0 and a uniform window give the
                 uniform capacity; window mean; clamps to [0, T]; monotone in the load
  swiglu         one-hot weights reduce each output to silu(a) * b closed form
  combine        grouped SwiGLU outputs combined equal layer_rows; hand example
  layer_rows     E=1, K=1 reduces to one dense SwiGLU; shared experts equal one
                 SwiGLU of concatenated width; dropped pairs contribute nothing
  balance        uniform routing gives exactly alpha
  router_zloss   all-equal logits give (l + ln E)^2
  utilization    uniform counts give log2 E bits (7 bits for 128 experts, the table's bound)
  flops          K=8, N_s=4, E=128 gives 12/128 (the compute-budget ratio)
  layer_backward central finite differences of the forward (layer_rows, select,
                 balance, router_zloss) with the routing held fixed, for every
                 input and weight element; offset gradients sum to zero
                 without the z-loss
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_LIB_OMP = os.path.join(_HERE, "libmoe_oracle_omp.so")

F64, F32, BF16 = 0, 1, 2
BIAS_PROB, BIAS_LOGIT = 0, 1


def build(force: bool = False, openmp: bool = False) -> str:
    """Compile moe_oracle.c with gcc (plain -O2: no fast-math, no reassociation);
    openmp: the -fopenmp build of the same source."""
    path = _LIB_OMP if openmp else _LIB
    if force or not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(_SRC):
        tmp = path + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", *(["-fopenmp"] if openmp else []),
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, path)
    return path


_libs = {}
_use_omp = False


def set_threads(n: int) -> int:
    """n == 1: the single-thread build (the default); n > 1: the OpenMP build
    on n threads.  Returns the threads the oracle now uses."""
    global _use_omp
    _use_omp = n > 1
    return int(_L().oracle_set_threads(n))


def _L():
    key = "omp" if _use_omp else "seq"
    if key not in _libs:
        lib = ctypes.CDLL(build(openmp=_use_omp))
        P = ctypes.c_void_p
        i64, i32, f32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_double
        lib.oracle_gate_logits.argtypes = [i64, i32, i32, P, i32, P, i32, P, P]
        lib.oracle_gate_logits.restype = None
        lib.oracle_softmax.argtypes = [i64, i32, P, P]
        lib.oracle_softmax.restype = None
        lib.oracle_select.argtypes = [i64, i32, i32, P, P, P, i32, P, P]
        lib.oracle_select.restype = ctypes.c_int
        lib.oracle_capacity.argtypes = [i64, i32, i32, f32]
        lib.oracle_capacity.restype = i64
        lib.oracle_dispatch.argtypes = [i64, i32, i32, i64, P, P, P, P, P, P]
        lib.oracle_dispatch.restype = ctypes.c_int
        lib.oracle_dispatch_caps.argtypes = [i64, i32, i32, P, P, P, P, P, P, P]
        lib.oracle_dispatch_caps.restype = ctypes.c_int
        lib.oracle_bias_update.argtypes = [i32, i64, P, P, f32, i32]
        lib.oracle_bias_update.restype = None
        lib.oracle_adaptive_capacity.argtypes = [i64, i32, i32, P, i32, f32, f32, P]
        lib.oracle_adaptive_capacity.restype = None
        lib.oracle_layer_backward.argtypes = [i64, i32, i32, i32, i32, i32, P, i32, P, P, P, P, P, i32,
                                              P, P, P, P, P, f64, P, f64, f64, P, P, P, P, P, P, P, P]
        lib.oracle_layer_backward.restype = ctypes.c_int
        lib.oracle_swiglu_accumulate.argtypes = [i32, i32, P, P, P, i32, f64, P, P]
        lib.oracle_swiglu_accumulate.restype = None
        lib.oracle_layer_rows.argtypes = [i64, i32, i32, i32, i32, i32, P, i32, P, P, P, P, i32,
                                          P, P, P, i64, P, P]
        lib.oracle_layer_rows.restype = ctypes.c_int
        lib.oracle_combine.argtypes = [i64, i32, i32, P, i32, P, P, P, i32, P]
        lib.oracle_combine.restype = None
        lib.oracle_balance.argtypes = [i64, i32, i32, P, P, f64, P, P, P]
        lib.oracle_balance.restype = None
        lib.oracle_router_zloss.argtypes = [i64, i32, P]
        lib.oracle_router_zloss.restype = f64
        lib.oracle_utilization.argtypes = [i32, P, P, P]
        lib.oracle_utilization.restype = None
        lib.oracle_flops.argtypes = [i64, i32, i32, i32, i32, i64, P]
        lib.oracle_flops.restype = None
        lib.oracle_set_threads.argtypes = [i32]
        lib.oracle_set_threads.restype = ctypes.c_int
        _libs[key] = lib
    return _libs[key]


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _as_input(a):
    """Return (contiguous array, type code) for an input tensor.

    Accepts float64 / float32 numpy arrays, or BF16 given as a uint16 numpy
    array of raw bits (or a torch.bfloat16 CPU tensor, viewed as such)."""
    if hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch  # local: only needed for torch inputs
        a = a.contiguous().view(torch.int16).numpy().view(np.uint16)
    elif hasattr(a, "numpy") and not isinstance(a, np.ndarray):
        a = a.contiguous().numpy()
    a = np.ascontiguousarray(a)
    if a.dtype == np.float64:
        return a, F64
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError(f"unsupported oracle input dtype {a.dtype}")


def gate_logits(x, w_gate, offset=None):
    """logits[t,e] = sum_j x[t,j] Wg[e,j] (+ offset[e]).

    Zen MoDE: Mixture of Distilled Experts Architecture, §3.1 Router
    Architecture (eq. router_standard: the linear projection W_r x)."""
    xa, xdt = _as_input(x)
    wa, wdt = _as_input(w_gate)
    T, d = xa.shape
    E = wa.shape[0]
    assert wa.shape == (E, d)
    off = None if offset is None else np.ascontiguousarray(offset, dtype=np.float32)
    out = np.empty((T, E), dtype=np.float64)
    _L().oracle_gate_logits(T, d, E, _ptr(xa), xdt, _ptr(wa), wdt, _ptr(off), _ptr(out))
    return out


def softmax(logits):
    """p = softmax over experts, per token (Zen MoDE §3.1, eq. router_standard)."""
    la = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = la.shape
    p = np.empty_like(la)
    _L().oracle_softmax(T, E, _ptr(la), _ptr(p))
    return p


def select(logits, K, bias=None, bias_mode=BIAS_PROB):
    """Top-K experts and renormalised gate weights.

    Selection score: the logit (no bias), p + b (Zen-Max §2.3
    Auxiliary-Loss-Free Load Balancing), or logit + b (BIAS_LOGIT variant).
    Ties go to the lower expert index.  Gate weights renormalise the selected
    probabilities to sum to one ("Scaling with experts", The gating network).
    Returns (idx [T,K] int32, w [T,K] float64, p [T,E] float64)."""
    la = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = la.shape
    p = softmax(la)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    idx = np.empty((T, K), dtype=np.int32)
    w = np.empty((T, K), dtype=np.float64)
    rc = _L().oracle_select(T, E, K, _ptr(la), _ptr(p), _ptr(b), int(bias_mode), _ptr(idx), _ptr(w))
    if rc != 0:
        raise ValueError("K must lie in [1, E]")
    return idx, w, p


def capacity(T, K, E, C):
    """ceil(C*T*K/E), or -1 for no limit (Zen MoDE §5.3, capacity_e; K-scaled)."""
    return int(_L().oracle_capacity(int(T), int(K), int(E), float(C)))


def dispatch(idx, E, cap):
    """Capacity-limited grouping of (token, k) pairs by expert ("Scaling with
    experts", A budget).  Returns dict of counts, kept, seg_off, slot_of, perm."""
    ia = np.ascontiguousarray(idx, dtype=np.int32)
    T, K = ia.shape
    counts = np.empty(E, np.int32)
    kept = np.empty(E, np.int32)
    seg_off = np.empty(E + 1, np.int32)
    slot_of = np.empty((T, K), np.int32)
    perm = np.full(max(T * K, 1), -1, np.int32)
    rc = _L().oracle_dispatch(T, K, E, int(cap), _ptr(ia), _ptr(counts), _ptr(kept), _ptr(seg_off),
                              _ptr(slot_of), _ptr(perm))
    if rc != 0:
        raise ValueError("expert index out of range")
    return dict(counts=counts, kept=kept, seg_off=seg_off, slot_of=slot_of,
                perm=perm[: int(seg_off[E])].copy())


def dispatch_caps(idx, E, caps):
    """dispatch() with one capacity per expert (caps[e] < 0: no limit), Zen MoDE
    §5.3 capacity_e per expert."""
    ia = np.ascontiguousarray(idx, dtype=np.int32)
    T, K = ia.shape
    ca = np.ascontiguousarray(caps, dtype=np.int64)
    assert ca.shape == (E,)
    counts = np.empty(E, np.int32)
    kept = np.empty(E, np.int32)
    seg_off = np.empty(E + 1, np.int32)
    slot_of = np.empty((T, K), np.int32)
    perm = np.full(max(T * K, 1), -1, np.int32)
    rc = _L().oracle_dispatch_caps(T, K, E, _ptr(ca), _ptr(ia), _ptr(counts), _ptr(kept), _ptr(seg_off),
                                   _ptr(slot_of), _ptr(perm))
    if rc != 0:
        raise ValueError("expert index out of range")
    return dict(counts=counts, kept=kept, seg_off=seg_off, slot_of=slot_of,
                perm=perm[: int(seg_off[E])].copy())


BIAS_UPDATE_SIGN, BIAS_UPDATE_PROPORTIONAL = 0, 1


def bias_update(counts, TK, bias, rate, mode=BIAS_UPDATE_SIGN):
    """One selection-bias update after a step (Zen-Max §2.3): overloaded experts'
    biases go down, underloaded ones' up.  Returns the new float32 biases."""
    c = np.ascontiguousarray(counts, dtype=np.int32)
    b = np.array(bias, dtype=np.float32, copy=True)
    assert b.shape == c.shape
    _L().oracle_bias_update(int(c.shape[0]), int(TK), _ptr(c), _ptr(b), float(rate), int(mode))
    return b


def adaptive_capacity(T, K, hist, c_base, gamma):
    """Per-expert capacities from the counts of the last n batches, hist [n, E]
    (Zen MoDE §5.3 Adaptive Capacity Factors).  Returns int64 [E]."""
    h = np.ascontiguousarray(hist, dtype=np.int32)
    n, E = h.shape
    caps = np.empty(E, np.int64)
    _L().oracle_adaptive_capacity(int(T), int(K), int(E), _ptr(h), int(n), float(c_base), float(gamma), _ptr(caps))
    return caps


def swiglu(x_row, w13, w2):
    """One SwiGLU expert on one token, (SiLU(x W_gate) * x W_up) W_down
    (Zen-Max §2.2 eq. Expert_i).  w13 [2F,d] (gate rows then up rows), w2 [d,F]."""
    xr = np.ascontiguousarray(x_row, dtype=np.float64)
    a, adt = _as_input(w13)
    b, bdt = _as_input(w2)
    assert adt == bdt
    d = xr.shape[0]
    F = a.shape[0] // 2
    h = np.empty(F, np.float64)
    out = np.zeros(d, np.float64)
    _L().oracle_swiglu_accumulate(d, F, _ptr(xr), _ptr(a), _ptr(b), adt, 1.0, _ptr(h), _ptr(out))
    return out


def layer_rows(x, w13, w2, idx, w, slot_of, rows=None, w13_shared=None, w2_shared=None):
    """Layer output for the listed tokens given the routing:
    y[t] = sum_s SharedExpert_s(x_t) + sum_{kept k} w[t,k] Expert_{idx[t,k]}(x_t)
    (Zen-Max §2.2; "Scaling with experts", The gating network / A budget /
    A shared expert).  Returns float64 [len(rows), d]."""
    xa, xdt = _as_input(x)
    a, wdt = _as_input(w13)
    b, bdt = _as_input(w2)
    assert wdt == bdt
    T, d = xa.shape
    E = a.shape[0]
    F = a.shape[1] // 2
    ia = np.ascontiguousarray(idx, dtype=np.int32)
    K = ia.shape[1]
    wa = np.ascontiguousarray(w, dtype=np.float64)
    sa = np.ascontiguousarray(slot_of, dtype=np.int32)
    if w13_shared is not None:
        ash, sdt = _as_input(w13_shared)
        bsh, sdt2 = _as_input(w2_shared)
        assert sdt == wdt and sdt2 == wdt
        ns = ash.shape[0]
    else:
        ash = bsh = None
        ns = 0
    r = np.arange(T, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    y = np.empty((r.shape[0], d), np.float64)
    rc = _L().oracle_layer_rows(T, d, E, K, F, ns, _ptr(xa), xdt, _ptr(a), _ptr(b), _ptr(ash), _ptr(bsh), wdt,
                                _ptr(ia), _ptr(wa), _ptr(sa), r.shape[0], _ptr(r), _ptr(y))
    if rc != 0:
        raise ValueError("token or expert index out of range")
    return y


def combine(y_perm, slot_of, w, y_shared=None):
    """y[t] = y_shared[t] + sum over kept k of w[t,k] * y_perm[slot_of[t,k]]
    ("Scaling with experts", The gating network / A budget / A shared expert).
    Returns float64 [T, d]."""
    ya, ydt = _as_input(y_perm)
    sa = np.ascontiguousarray(slot_of, dtype=np.int32)
    wa = np.ascontiguousarray(w, dtype=np.float64)
    T, K = sa.shape
    d = ya.shape[1]
    if y_shared is not None:
        sh, sdt = _as_input(y_shared)
    else:
        sh, sdt = None, F64
    y = np.empty((T, d), np.float64)
    _L().oracle_combine(T, d, K, _ptr(ya), ydt, _ptr(sa), _ptr(wa), _ptr(sh), sdt, _ptr(y))
    return y


def balance(counts, p, K, alpha=0.01):
    """Switch statistics f_e, P_e and L = alpha*E*sum f_e P_e (Zen MoDE §5.2
    eq. L_balance; "Scaling with experts", A balance penalty).
    Returns (f [E], P [E], loss)."""
    ca = np.ascontiguousarray(counts, dtype=np.int32)
    pa = np.ascontiguousarray(p, dtype=np.float64)
    T, E = pa.shape
    f = np.empty(E, np.float64)
    P = np.empty(E, np.float64)
    loss = ctypes.c_double(0.0)
    _L().oracle_balance(T, E, int(K), _ptr(ca), _ptr(pa), float(alpha), _ptr(f), _ptr(P), ctypes.byref(loss))
    return f, P, loss.value


def router_zloss(logits):
    """(1/B) sum_x (logsumexp x)^2 (Zen-Max §3.2, router z-loss)."""
    la = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = la.shape
    return float(_L().oracle_router_zloss(T, E, _ptr(la)))


def utilization(counts, kept):
    """Entropy (bits), CV, drop rate, #experts < 50% and > 200% of the mean
    load (Zen MoDE §6.2, table tab:utilization)."""
    ca = np.ascontiguousarray(counts, dtype=np.int32)
    ka = np.ascontiguousarray(kept, dtype=np.int32)
    out = np.empty(5, np.float64)
    _L().oracle_utilization(ca.shape[0], _ptr(ca), _ptr(ka), _ptr(out))
    return dict(entropy_bits=out[0], cv=out[1], drop_rate=out[2],
                n_below_half=int(out[3]), n_above_double=int(out[4]))


def flops(T, d, E, F, n_shared, kept_pairs):
    """Algorithmic FLOPs (router, experts) and the expert/dense-equivalent
    ratio (Zen MoDE §7.1 Compute Budget).  Returns (total, expert, ratio)."""
    out = np.empty(3, np.float64)
    _L().oracle_flops(int(T), int(d), int(E), int(F), int(n_shared), int(kept_pairs), _ptr(out))
    return float(out[0]), float(out[1]), float(out[2])


def layer_backward(x, wg, w13, w2, logits, idx, w, slot_of, counts, alpha, dy, c_bal=1.0, c_z=0.0,
                   w13_shared=None, w2_shared=None):
    """Gradients of the layer for training (routing held fixed): dJ/dy = dy,
    dJ/dL_balance = c_bal, dJ/dL_z = c_z.  Zen-Max §2.2 (experts), "Scaling with
    experts" (The gating network, A balance penalty), Zen-Max §3.2 (z-loss).
    Returns float64 arrays dx, dw13, dw2, dw13_shared, dw2_shared, dwg, doff, dlogits."""
    xa, xdt = _as_input(x)
    ga, gdt = _as_input(wg)
    a, wdt = _as_input(w13)
    b, bdt = _as_input(w2)
    assert gdt == wdt == bdt
    T, d = xa.shape
    E, F2, _ = a.shape
    F = F2 // 2
    K = np.asarray(idx).shape[1]
    Ns = 0 if w13_shared is None else np.asarray(w13_shared).shape[0]
    sa = sb = None
    if Ns:
        sa, sdt = _as_input(w13_shared)
        sb, _ = _as_input(w2_shared)
        assert sdt == wdt
    la = np.ascontiguousarray(logits, dtype=np.float64)
    ia = np.ascontiguousarray(idx, dtype=np.int32)
    wa = np.ascontiguousarray(w, dtype=np.float64)
    so = np.ascontiguousarray(slot_of, dtype=np.int32)
    ca = np.ascontiguousarray(counts, dtype=np.int32)
    dya = np.ascontiguousarray(dy, dtype=np.float64)
    out = dict(dx=np.empty((T, d)), dw13=np.empty((E, 2 * F, d)), dw2=np.empty((E, d, F)),
               dw13_shared=np.empty((Ns, 2 * F, d)), dw2_shared=np.empty((Ns, d, F)), dwg=np.empty((E, d)),
               doff=np.empty(E), dlogits=np.empty((T, E)))
    rc = _L().oracle_layer_backward(T, d, E, K, F, Ns, _ptr(xa), xdt, _ptr(ga), _ptr(a), _ptr(b), _ptr(sa), _ptr(sb),
                                    wdt, _ptr(la), _ptr(ia), _ptr(wa), _ptr(so), _ptr(ca), float(alpha), _ptr(dya),
                                    float(c_bal), float(c_z), _ptr(out["dx"]), _ptr(out["dw13"]), _ptr(out["dw2"]),
                                    _ptr(out["dw13_shared"]), _ptr(out["dw2_shared"]), _ptr(out["dwg"]),
                                    _ptr(out["doff"]), _ptr(out["dlogits"]))
    if rc != 0:
        raise ValueError("expert index out of range")
    return out
