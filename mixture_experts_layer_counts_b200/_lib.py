"""ctypes binding of ``libmoe.so`` (the C ABI declared in include/moe.h).

Argument marshalling only: every step of the layer runs in the CUDA library.
There is no fallback: if the library is missing the import of this module's
functions raises.
"""
from __future__ import annotations

import ctypes as C
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_DTYPE_BF16 = 0
MOE_DTYPE_FP8_E4M3 = 1

STATUS = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
    3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_TIMEOUT",
    6: "MOE_ERR_DEVICE_BOUNDS", 7: "MOE_ERR_MISALIGNED", 8: "MOE_ERR_EXCEEDS_STATIC_SCRATCH",
}

# every symbol include/moe.h declares
EXPORTS = ("moe_workspace_size", "moe_workspace_init", "moe_forward", "moe_forward_hostio",
           "moe_route", "moe_align", "moe_get_status", "moe_status_string", "moe_route_static",
           "moe_forward_batch_invariant", "moe_cache_stats", "moe_forward_partial", "moe_sum_partials",
           "moe_inv_rope_fp8_quant")


class DebugOut(C.Structure):
    _fields_ = [
        ("topk_ids", C.c_void_p), ("topk_w", C.c_void_p), ("counts", C.c_void_p),
        ("offsets", C.c_void_p), ("perm", C.c_void_p), ("inv_perm", C.c_void_p),
        ("inter", C.c_void_p), ("act_scales", C.c_void_p), ("stage_events", C.c_void_p),
        ("force_orient", C.c_int), ("wait_timeout_us", C.c_int), ("inject_stall", C.c_int),
        ("hidden_q", C.c_void_p),
    ]


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


_lib = None


def lib() -> C.CDLL:
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m mixture_experts_layer_counts_b200.build`")
        L = C.CDLL(LIB_PATH)
        vp, i, sz = C.c_void_p, C.c_int, C.c_size_t
        L.moe_workspace_size.restype = sz
        L.moe_workspace_size.argtypes = [i] * 6
        L.moe_workspace_init.restype = i
        L.moe_workspace_init.argtypes = [vp, sz, vp]
        L.moe_forward.restype = i
        L.moe_forward.argtypes = [vp] * 7 + [i] * 6 + [vp, vp, sz, C.POINTER(DebugOut), vp]
        L.moe_forward_batch_invariant.restype = i
        L.moe_forward_batch_invariant.argtypes = [vp] * 5 + [i] * 5 + [vp, vp, sz, vp, vp]
        L.moe_forward_hostio.restype = i
        L.moe_forward_hostio.argtypes = [vp] * 7 + [i] * 6 + [vp, vp, sz, vp]
        L.moe_forward_partial.restype = i
        L.moe_forward_partial.argtypes = [vp] * 7 + [i] * 6 + [vp, vp, sz, vp]
        L.moe_sum_partials.restype = i
        L.moe_sum_partials.argtypes = [vp, i, i, i, vp, vp]
        L.moe_inv_rope_fp8_quant.restype = i
        L.moe_inv_rope_fp8_quant.argtypes = [vp] * 4 + [i] * 4 + [vp, vp, vp]
        L.moe_route.restype = i
        L.moe_route.argtypes = [vp, vp, vp, i, i, i, i, vp, vp, vp, sz, vp]
        L.moe_route_static.restype = i
        L.moe_route_static.argtypes = [vp, vp, vp, i, i, i, i, vp, vp, vp]
        L.moe_align.restype = i
        L.moe_align.argtypes = [vp, i, i, i, vp, vp, vp, vp, vp, sz, vp]
        L.moe_get_status.restype = i
        L.moe_get_status.argtypes = [vp, vp, C.POINTER(C.c_uint32)]
        L.moe_cache_stats.restype = None
        L.moe_cache_stats.argtypes = [C.POINTER(C.c_ulonglong)]
        L.moe_status_string.restype = C.c_char_p
        L.moe_status_string.argtypes = [i]
        _lib = L
    return _lib


def check(code: int, where: str) -> None:
    if code != 0:
        raise MoEError(code, where)
