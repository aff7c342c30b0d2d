"""ctypes loader of libmoe_b200.so (the C ABI declared in include/moe.h).

There is no fallback: if the shared library is missing or cannot be loaded this module
raises, so a product call can never silently run anything but the CUDA kernels.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libmoe_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "moe.h")

MOE_OK = 0
MOE_ERR_ARG = -1
MOE_ERR_SHAPE = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4
MOE_ERR_UNIMPLEMENTED = -5
MOE_ERR_DEVICE = -6

MOE_SOFTMAX = 0
MOE_SIGMOID = 1
MOE_SQRTSOFTPLUS = 2

MOE_ST_NAN_TOKENS = 0
MOE_ST_ZERO_DENOM = 1
MOE_ST_BAD_EXPERT_ID = 2
MOE_ST_PIPE_TIMEOUT = 3
MOE_STATUS_WORDS = 8

MOE_STAGE_ROUTE = 0
MOE_STAGE_PERMUTE = 1
MOE_STAGE_FFN = 2
MOE_STAGE_COMBINE = 3
MOE_STAGE_FORWARD = 4
MOE_STAGE_STATS = 5
MOE_STAGE_BACKWARD = 6
MOE_NUM_STAGE_EVENTS = 8


class MoeCfg(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("E", ctypes.c_int32),
                ("K", ctypes.c_int32), ("I", ctypes.c_int32), ("I_shared", ctypes.c_int32),
                ("score_fn", ctypes.c_int32), ("renorm", ctypes.c_int32),
                ("route_scale", ctypes.c_float), ("n_group", ctypes.c_int32),
                ("topk_group", ctypes.c_int32)]


_P = ctypes.c_void_p
_SZ = ctypes.c_size_t
_CFG = ctypes.POINTER(MoeCfg)
_I = ctypes.c_int

SIGNATURES = {
    "moe_workspace_bytes": (_SZ, [_CFG, _I]),
    "moe_route": (_I, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_permute": (_I, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_permute_noalloc": (_I, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_grouped_ffn": (_I, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_combine": (_I, [_CFG, _P, _P, _P, _P, _P, _P, _P]),
    "moe_combine_invariant": (_I, [_CFG, _P, _P, _P, _P, _P, _P, _P]),
    "moe_forward": (_I, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                         _SZ, _P, _P]),
    "moe_router_stats": (_I, [_CFG, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_backward": (_I, [_CFG] + [_P] * 19 + [_I, _P, _P, _SZ, _P]),
    "moe_forward_train": (_I, [_CFG] + [_P] * 15 + [_SZ, _P]),
    "moe_forward_host_workspace_bytes": (_SZ, [_CFG, _I]),
    "moe_forward_host": (_I, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _SZ, _P]),
    "moe_status_string": (ctypes.c_char_p, [_I]),
    "moe_abi_version": (_I, []),
    "moe_pipeline_wait_selftest": (_I, [_P, ctypes.c_longlong, _P]),
}

_lock = threading.Lock()
_lib = None


def load():
    """The loaded library (raises if it is not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"libmoe_b200.so is not built ({LIB_PATH}); run "
                    "`python -m deterministic_invariant_routing_b200.build` (needs nvcc)")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(lib, name)
                f.restype = res
                f.argtypes = args
            _lib = lib
    return _lib


def status_string(code: int) -> str:
    return load().moe_status_string(code).decode()
