"""ctypes binding of libmoe.so (include/moe.h).  Marshalling only.

The library is loaded from this package's directory.  There is no fallback:
if the shared object is missing the import fails with the build command.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

# moe_status
MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_INVALID_TOPK = 2
MOE_ERR_CAPACITY_TOO_TIGHT = 3
MOE_ERR_UNSUPPORTED = 4
MOE_ERR_WORKSPACE = 5
MOE_ERR_CUDA = 6
MOE_ERR_DEVICE = 7
# moe_phase
MOE_PHASE_START, MOE_PHASE_ROUTE, MOE_PHASE_PERMUTE, MOE_PHASE_FFN1, MOE_PHASE_FFN2, MOE_PHASE_SHARED, \
    MOE_PHASE_COMBINE, MOE_PHASE_COUNT = range(8)
# moe_ws_region
MOE_WS_OFFSETS, MOE_WS_PERM_TOKEN, MOE_WS_PERM_W, MOE_WS_SLOT_ROW, MOE_WS_X_PERM, MOE_WS_H, MOE_WS_Y_PERM, \
    MOE_WS_SHARED_H, MOE_WS_SHARED_OUT, MOE_WS_ROUTER_LOGITS, MOE_WS_REGION_COUNT = range(11)
# moe_router_kind
MOE_ROUTER_SOFTMAX_TOPK = 0
MOE_ROUTER_SIGMOID_GROUP = 1
# moe_act
MOE_ACT_RELU = 0
MOE_ACT_SWIGLU = 1
# moe_dtype
MOE_F32 = 0
MOE_BF16 = 1
MOE_Q4_AFFINE_G64 = 2
# moe_weight_layout
MOE_LAYOUT_SEPARATE = 0
MOE_LAYOUT_FUSED_GATE_UP = 1


class moe_config(C.Structure):
    _fields_ = [
        ("num_tokens", C.c_int32),
        ("hidden", C.c_int32),
        ("intermediate", C.c_int32),
        ("num_experts", C.c_int32),
        ("top_k", C.c_int32),
        ("router", C.c_int32),
        ("norm_topk_prob", C.c_int32),
        ("routed_scaling", C.c_float),
        ("n_group", C.c_int32),
        ("topk_group", C.c_int32),
        ("capacity_factor", C.c_float),
        ("act", C.c_int32),
        ("act_dtype", C.c_int32),
        ("weight_dtype", C.c_int32),
        ("shared_intermediate", C.c_int32),
        ("aux_alpha", C.c_float),
        ("weight_layout", C.c_int32),
        ("fused_gather", C.c_int32),
    ]


class moe_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in (
        "w1", "w2", "w3", "scale1", "scale2", "scale3", "bias1", "bias2", "bias3",
        "shared1", "shared2", "shared3")]


class moe_stats(C.Structure):
    _fields_ = [("raw_counts", C.c_void_p), ("kept_counts", C.c_void_p),
                ("prob_sum", C.c_void_p), ("dropped", C.c_void_p)]


_P = C.c_void_p
_CFG = C.POINTER(moe_config)
_W = C.POINTER(moe_weights)
_S = C.POINTER(moe_stats)

# name -> (restype, argtypes)
SIGNATURES = {
    "moe_capacity": (C.c_int64, [C.c_int32, C.c_int32, C.c_int32, C.c_float]),
    "moe_validate": (C.c_int, [_CFG]),
    "moe_workspace_size": (C.c_size_t, [_CFG]),
    "moe_aux_loss": (C.c_int, [_CFG, _P, _P, C.POINTER(C.c_double), C.POINTER(C.c_double)]),
    "moe_routing_health": (C.c_int, [_CFG, _P, C.c_int32, C.POINTER(C.c_double), C.POINTER(C.c_double),
                                     C.POINTER(C.c_double), C.POINTER(C.c_int32)]),
    "moe_status_string": (C.c_char_p, [C.c_int]),
    "moe_last_error": (C.c_char_p, []),
    "moe_kernel_launches": (C.c_int64, []),
    "moe_set_wait_timeout_ns": (C.c_int, [C.c_uint64]),
    "moe_workspace_status": (C.c_int, [_P, _P]),
    "moe_set_phase_events": (C.c_int, [C.POINTER(C.c_void_p), C.c_int32]),
    "moe_workspace_region": (C.c_int, [_CFG, C.c_int32, C.POINTER(C.c_size_t), C.POINTER(C.c_size_t)]),
    "moe_route": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, C.c_size_t, _P]),
    "moe_route_noalloc": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P]),
    "moe_route_forced": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, C.c_size_t, _P]),
    "moe_update_bias": (C.c_int, [_CFG, _P, _P, C.c_float, _P]),
    "moe_permute": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P, C.c_size_t, _P]),
    "moe_expert_counts": (C.c_int, [_CFG, _P, _P, _P, C.c_size_t, _P]),
    "moe_permute_shard": (C.c_int, [_CFG, _P, _P, _P, _P, C.c_int32, C.c_int32, C.c_int64, _P, _P, _P, _P, _P, _S,
                                    _P, C.c_size_t, _P]),
    "moe_ep_local_ids": (C.c_int, [_P, C.c_int32, C.c_int32, C.c_int32, _P, _P]),
    "moe_grouped_ffn": (C.c_int, [_CFG, _P, _P, _W, _P, _P, C.c_size_t, _P]),
    "moe_shared_expert": (C.c_int, [_CFG, _P, _W, _P, _P, C.c_size_t, _P]),
    "moe_combine": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P]),
    "moe_forward": (C.c_int, [_CFG, _P, _P, _P, _W, _P, _P, _P, _S, _P, C.c_size_t, _P]),
    "moe_forward_host": (C.c_int, [_CFG, _P, _P, _P, _W, _P, _P, _P, _P, _P, C.c_size_t, _P]),
}

_lib = None


def lib() -> C.CDLL:
    """The loaded library (loaded once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m mixture_experts_layer_41_b200.build` (there is no CPU fallback)")
        handle = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        text = lib().moe_status_string(status).decode()
        detail = lib().moe_last_error().decode()
        msg = f"{where}: {text} (status {status})"
        if status in (MOE_ERR_CUDA, MOE_ERR_DEVICE) and detail:
            msg += f": {detail}"
        super().__init__(msg)


def check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoEError(status, where)
