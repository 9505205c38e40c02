"""ctypes binding of libmoe.so (declarations in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Loading fails loudly when libmoe.so is missing; there is no
fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_OK, MOE_ERR_ARG, MOE_ERR_CUDA, MOE_ERR_DEVICE, MOE_ERR_TIMEOUT = 0, -1, -2, -3, -4
MOE_FP32, MOE_BF16 = 0, 1
MOE_SOFTMAX, MOE_SIGMOID = 0, 1
MOE_GMAX, MOE_GTOP2SUM = 0, 1
MOE_GEMM_AUTO, MOE_GEMM_SIMT = 0, 1
DEVERR_EXPERT_ID, DEVERR_TIMEOUT, DEVERR_ROWS = 1, 2, 4

c_int32, c_int64, c_float, c_void_p = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p

# every symbol include/moe.h declares
EXPORTS = ("moe_get_sizes", "moe_router", "moe_dispatch", "moe_aux_loss",
           "moe_expert_ffn", "moe_combine", "moe_backward", "moe_check_status",
           "moe_status_string", "moe_last_cuda_error", "moe_launch_count",
           "moe_profile_enable", "moe_profile_reset", "moe_profile_read", "moe_profile_starts",
           "moe_profile_name", "moe_profile_side", "moe_profile_disable",
           "moe_dispatch_static", "moe_set_side_streams", "moe_aux_loss_seq",
           "moe_bias_update", "moe_route_expert_choice", "moe_expert_ffn_gather",
           "moe_expert_ffn_combine", "moe_aux_stats", "moe_aux_loss_global",
           "moe_set_backward_streams")


class MoeConfig(ctypes.Structure):
    _fields_ = [("T", c_int32), ("D", c_int32), ("E", c_int32), ("K", c_int32),
                ("F", c_int32), ("n_shared", c_int32), ("dtype", c_int32),
                ("score_fn", c_int32), ("renorm", c_int32), ("n_groups", c_int32),
                ("topk_groups", c_int32), ("group_score", c_int32),
                ("capacity_factor", c_float), ("min_capacity", c_int32),
                ("route_scale", c_float), ("aux_alpha", c_float),
                ("z_lambda", c_float), ("gemm_impl", c_int32), ("seq_len", c_int32),
                ("expert_choice", c_int32), ("loss_tokens", c_int32),
                ("expert_base", c_int32), ("n_local_experts", c_int32)]


class MoeSizes(ctypes.Structure):
    _fields_ = [("rows_max", c_int64), ("tiles_max", c_int64),
                ("capacity", c_int64), ("ws_bytes", ctypes.c_size_t),
                ("row_align", c_int64)]


class MoEError(RuntimeError):
    pass


_lib = None


def lib():
    """The loaded libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            "libmoe.so not found at %s: build it with "
            "`python -m mixture_experts_routing_fp32_b200.build`" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    P = c_void_p
    cfg = ctypes.POINTER(MoeConfig)
    sig = {
        "moe_get_sizes": [cfg, ctypes.POINTER(MoeSizes)],
        "moe_router": [cfg, P, P, P, P, P, P, P, P, P, P, P, P],
        "moe_dispatch": [cfg, P, P, P, P, P, P, P, P, P, P, P, P, P],
        "moe_aux_loss": [cfg, P, P, P, P, P, P],
        "moe_expert_ffn": [cfg, P, P, P, P, P, P, P, P, P, P, P, P, P],
        "moe_expert_ffn_gather": [cfg] + [P] * 14,
        "moe_expert_ffn_combine": [cfg] + [P] * 18,
        "moe_combine": [cfg, P, P, P, P, P, P],
        "moe_backward": [cfg] + [P] * 33,
        "moe_check_status": [P, ctypes.POINTER(ctypes.c_uint32)],
        "moe_status_string": [ctypes.c_int],
        "moe_last_cuda_error": [],
        "moe_launch_count": [ctypes.c_int],
        "moe_profile_enable": [ctypes.c_int],
        "moe_set_side_streams": [ctypes.c_int],
        "moe_profile_reset": [],
        "moe_profile_read": [ctypes.POINTER(ctypes.c_float), ctypes.c_int],
        "moe_profile_starts": [ctypes.POINTER(ctypes.c_float), ctypes.c_int],
        "moe_profile_name": [ctypes.c_int],
        "moe_profile_side": [ctypes.c_int],
        "moe_profile_disable": [],
        "moe_dispatch_static": [cfg, P, P, P, P, P, P, P, P, P, P, P, P],
        "moe_aux_loss_seq": [cfg, P, P, P, P, P, P, P],
        "moe_bias_update": [cfg, P, P, ctypes.c_float, P],
        "moe_route_expert_choice": [cfg] + [P] * 12,
        "moe_aux_stats": [cfg, P, P, P, P, P],
        "moe_aux_loss_global": [cfg, P, P, P, P],
        "moe_set_backward_streams": [P],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_launch_count.restype = ctypes.c_int64
    L.moe_profile_name.restype = ctypes.c_char_p
    _lib = L
    return L


def check(rc: int, what: str):
    if rc != MOE_OK:
        L = lib()
        msg = L.moe_status_string(rc).decode()
        if rc == MOE_ERR_CUDA:
            msg += " (cudaError %d)" % L.moe_last_cuda_error()
        raise MoEError("%s failed: %s [%d]" % (what, msg, rc))
