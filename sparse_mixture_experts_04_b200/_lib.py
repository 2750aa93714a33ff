"""ctypes view of libmoe_b200.so (the C ABI in include/moe_b200.h).

Loading fails loudly when the library has not been built: there is no other
implementation of the layer to fall back to.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_CUDA",
                -4: "MOE_ERR_DEVICE_CHECK", -5: "MOE_ERR_WORKSPACE"}
DTYPE_BF16, DTYPE_F32 = 0, 1
FLAG_LOGITS_GIVEN, FLAG_BIAS_LOGIT, FLAG_EXTENDED_STATS, FLAG_EXPERT_CAPACITY = 0x1, 0x2, 0x4, 0x8
FLAG_SAVE_GU = 0x10
BIAS_UPDATE_SIGN, BIAS_UPDATE_PROPORTIONAL = 0, 1
ABI_VERSION = 2
EXTENDED_STATS = ("z_loss", "entropy_bits", "cv", "drop_rate", "n_below_half", "n_above_double")
FFN_ROUTED, FFN_SHARED = 0, 1
DEV_BAD_EXPERT, DEV_WAIT_TIMEOUT = 0x1, 0x2

# every symbol include/moe_b200.h declares
EXPORTED = ("moe_abi_version", "moe_status_string", "moe_capacity", "moe_max_rows", "moe_workspace_size",
            "moe_reset_device_status", "moe_read_device_status", "moe_route", "moe_dispatch",
            "moe_expert_ffn", "moe_combine", "moe_layer_forward", "moe_layer_forward_profiled",
            "moe_layer_forward_clocked", "moe_expert_ffn_segments",
            "moe_dispatch_noalloc", "moe_dispatch_capacity", "moe_balance_update", "moe_backward_workspace_size",
            "moe_layer_backward", "moe_ep_plan", "moe_ep_peer_plan", "moe_ep_scatter", "moe_ep_combine",
            "moe_ipc_malloc", "moe_ipc_free", "moe_ipc_handle", "moe_ipc_open", "moe_ipc_close")
NUM_EVENTS = 7  # MOE_EV_START .. MOE_EV_END
EVENT_NAMES = ("start", "routed", "dispatched", "up", "down", "shared", "end")
NUM_CLOCKS = 7  # MOE_CLOCK_ROUTE .. MOE_CLOCK_COMBINE
CLOCK_NAMES = ("route", "dispatch", "gather", "up", "down", "shared", "combine")


class MoeProblem(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d_model", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("dtype", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("alpha", ctypes.c_float)]


class MoeWeights(ctypes.Structure):
    _fields_ = [("w_gate", ctypes.c_void_p), ("logit_offset", ctypes.c_void_p), ("sel_bias", ctypes.c_void_p),
                ("w13", ctypes.c_void_p), ("w2", ctypes.c_void_p), ("w13_shared", ctypes.c_void_p),
                ("w2_shared", ctypes.c_void_p), ("expert_capacity", ctypes.c_void_p)]


class MoeRouting(ctypes.Structure):
    _fields_ = [("logits", ctypes.c_void_p), ("topk_idx", ctypes.c_void_p), ("topk_w", ctypes.c_void_p),
                ("counts", ctypes.c_void_p), ("kept", ctypes.c_void_p), ("seg_off", ctypes.c_void_p),
                ("slot_of", ctypes.c_void_p), ("perm", ctypes.c_void_p)]


class MoeGrads(ctypes.Structure):
    _fields_ = [("dx", ctypes.c_void_p), ("dw13", ctypes.c_void_p), ("dw2", ctypes.c_void_p),
                ("dw13_shared", ctypes.c_void_p), ("dw2_shared", ctypes.c_void_p), ("dw_gate", ctypes.c_void_p),
                ("d_offset", ctypes.c_void_p), ("d_logits", ctypes.c_void_p)]


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} returned {code} ({STATUS_NAMES.get(code, 'unknown')})")


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m sparse_mixture_experts_04_b200.build` "
                           "(the layer has no other implementation)")
    L = ctypes.CDLL(LIB_PATH)
    P, PP = ctypes.c_void_p, ctypes.POINTER(MoeProblem)
    i32, i64, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    L.moe_abi_version.argtypes, L.moe_abi_version.restype = [], ctypes.c_int
    L.moe_status_string.argtypes, L.moe_status_string.restype = [ctypes.c_int], ctypes.c_char_p
    L.moe_capacity.argtypes, L.moe_capacity.restype = [PP], i64
    L.moe_max_rows.argtypes, L.moe_max_rows.restype = [PP], i64
    L.moe_workspace_size.argtypes, L.moe_workspace_size.restype = [PP, ctypes.POINTER(sz)], ctypes.c_int
    L.moe_reset_device_status.argtypes, L.moe_reset_device_status.restype = [P, P], ctypes.c_int
    L.moe_read_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
    L.moe_read_device_status.restype = ctypes.c_int
    L.moe_route.argtypes = [PP, P, P, P, P, P, P, P, P, P, sz, P]
    L.moe_route.restype = ctypes.c_int
    L.moe_dispatch.argtypes = [PP, P, P, P, P, P, P, P, P, P, sz, P]
    L.moe_dispatch.restype = ctypes.c_int
    L.moe_expert_ffn.argtypes = [PP, i32, P, i64, P, P, P, P, P, sz, P]
    L.moe_expert_ffn.restype = ctypes.c_int
    L.moe_expert_ffn_segments.argtypes = [PP, P, i64, P, i32, P, P, P, P, sz, P]
    L.moe_expert_ffn_segments.restype = ctypes.c_int
    L.moe_combine.argtypes = [PP, P, P, P, P, P, P, sz, P]
    L.moe_combine.restype = ctypes.c_int
    L.moe_layer_forward.argtypes = [PP, P, ctypes.POINTER(MoeWeights), P, ctypes.POINTER(MoeRouting), P, P, sz, P]
    L.moe_layer_forward.restype = ctypes.c_int
    L.moe_layer_forward_profiled.argtypes = [PP, P, ctypes.POINTER(MoeWeights), P, ctypes.POINTER(MoeRouting), P,
                                             P, sz, P, ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(i32)]
    L.moe_layer_forward_profiled.restype = ctypes.c_int
    L.moe_layer_forward_clocked.argtypes = [PP, P, ctypes.POINTER(MoeWeights), P, ctypes.POINTER(MoeRouting), P,
                                            P, sz, P, P]
    L.moe_layer_forward_clocked.restype = ctypes.c_int
    L.moe_dispatch_noalloc.argtypes = [PP, P, P, P, P, P, P, P, P, P]
    L.moe_dispatch_noalloc.restype = ctypes.c_int
    L.moe_dispatch_capacity.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, sz, P]
    L.moe_dispatch_capacity.restype = ctypes.c_int
    L.moe_balance_update.argtypes = [PP, P, P, ctypes.c_float, i32, P, i32, i64, ctypes.c_float, ctypes.c_float,
                                     P, P]
    L.moe_balance_update.restype = ctypes.c_int
    L.moe_backward_workspace_size.argtypes = [PP, ctypes.POINTER(sz)]
    L.moe_backward_workspace_size.restype = ctypes.c_int
    L.moe_layer_backward.argtypes = [PP, P, ctypes.POINTER(MoeWeights), ctypes.POINTER(MoeRouting), P, sz, P,
                                     ctypes.c_float, ctypes.c_float, ctypes.POINTER(MoeGrads), P, sz, P]
    L.moe_layer_backward.restype = ctypes.c_int
    L.moe_ep_plan.argtypes = [i32, i32, i32, P, P, P, P]
    L.moe_ep_plan.restype = ctypes.c_int
    L.moe_ep_peer_plan.argtypes = [i32, i32, i32, P, P, P, P]
    L.moe_ep_peer_plan.restype = ctypes.c_int
    L.moe_ep_scatter.argtypes = [PP, i32, P, P, P, P, P, P]
    L.moe_ep_scatter.restype = ctypes.c_int
    L.moe_ep_combine.argtypes = [PP, i32, P, P, P, P, P, P, P, P]
    L.moe_ep_combine.restype = ctypes.c_int
    L.moe_ipc_malloc.argtypes = [sz, ctypes.POINTER(ctypes.c_void_p)]
    L.moe_ipc_malloc.restype = ctypes.c_int
    L.moe_ipc_free.argtypes = [P]
    L.moe_ipc_free.restype = ctypes.c_int
    L.moe_ipc_handle.argtypes = [P, P]
    L.moe_ipc_handle.restype = ctypes.c_int
    L.moe_ipc_open.argtypes = [P, ctypes.POINTER(ctypes.c_void_p)]
    L.moe_ipc_open.restype = ctypes.c_int
    L.moe_ipc_close.argtypes = [P]
    L.moe_ipc_close.restype = ctypes.c_int
    if L.moe_abi_version() != ABI_VERSION:
        raise RuntimeError(f"{LIB_PATH} has ABI version {L.moe_abi_version()}, this binding expects {ABI_VERSION}: "
                           "rebuild it")
    _lib = L
    return L


def check(fn: str, rc: int) -> None:
    if rc != MOE_OK:
        raise MoeError(fn, rc)
