"""ctypes loader of ``libmoe_mxfp4.so`` (the sm_100a C-ABI library).

There is no fallback: if the library cannot be built or loaded, importing the
binding raises. PyTorch supplies device memory and streams only.
"""
from __future__ import annotations

import ctypes as C
import os

from . import build as _build

_L = None

MOE_OK = 0
STATUS_NAMES = {
    0: "MOE_OK", -1: "MOE_ERR_ARG", -2: "MOE_ERR_NOT_LOADED", -3: "MOE_ERR_NOT_DEVICE",
    -4: "MOE_ERR_ALIGN", -5: "MOE_ERR_WORKSPACE", -6: "MOE_ERR_CUDA",
    -7: "MOE_ERR_DEVICE_STATUS", -8: "MOE_ERR_UNSUPPORTED",
}

# (name, restype, argtypes) of every exported symbol of include/moe_mxfp4.h
_vp, _i, _u, _sz, _i64 = C.c_void_p, C.c_int, C.c_uint, C.c_size_t, C.c_int64
SIGNATURES = [
    ("moe_create", _i, [_i, _i, _i, _i, C.POINTER(_vp)]),
    ("moe_destroy", _i, [_vp]),
    ("moe_load_packed", _i, [_vp, _vp, _vp]),
    ("moe_load_packed_nvfp4", _i, [_vp, _vp, _vp, _vp]),
    ("moe_load_packed_sym8", _i, [_vp, _vp, _vp]),
    ("moe_load_expert_table", _i, [_vp, C.POINTER(_vp), C.POINTER(_vp)]),
    ("moe_workspace_bytes", _i, [_vp, _i, C.POINTER(_sz)]),
    ("moe_set_workspace", _i, [_vp, _vp, _sz, _i]),
    ("moe_route", _i, [_vp, _vp, _i, _vp, _vp, _vp, _vp, _vp]),
    ("moe_route_ex", _i, [_vp, _vp, _i, _vp, _vp, _u, _vp, _vp, _vp, _vp, _vp]),
    ("moe_forward", _i, [_vp, _vp, _i, _vp, _vp, _vp, _vp]),
    ("moe_forward_ex", _i, [_vp, _vp, _i, _vp, _vp, _vp, _vp, _u, _vp]),
    ("moe_layer_ex", _i, [_vp, _vp, _i, _vp, _vp, _u, _vp, _vp, _vp, _vp, _vp, _vp, _u, _vp]),
    ("moe_get_intermediates", _i, [_vp, C.POINTER(_vp), C.POINTER(_vp)]),
    ("moe_get_status", _i, [_vp, C.POINTER(_u)]),
    ("moe_get_status_stream", _i, [_vp, _vp, C.POINTER(_u)]),
    ("moe_bytes_per_expert", _i, [_vp, C.POINTER(_sz)]),
    ("moe_set_tuning", _i, [_vp, _i, _i]),
    ("moe_set_fusion", _i, [_vp, _i]),
    ("moe_status_string", C.c_char_p, [_i]),
    ("moe_device_check", _i, []),
    ("moe_debug_dequant", _i, [_vp, _vp, _i64, _vp, _vp]),
    ("moe_forward_noalloc", _i, [_i, _i, _i, _i, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp]),
    ("moe_forward_noalloc_status", _i, [_vp, C.POINTER(_u)]),
    ("moe_stack_create", _i, [C.POINTER(_vp), _i, C.POINTER(_vp), C.POINTER(_vp), C.POINTER(_vp)]),
    ("moe_stack_destroy", _i, [_vp]),
    ("moe_stack_workspace_bytes", _i, [_vp, C.POINTER(_sz)]),
    ("moe_stack_set_workspace", _i, [_vp, _vp, _sz]),
    ("moe_stack_decode", _i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    ("moe_stack_get_status", _i, [_vp, _vp, C.POINTER(_u)]),
    ("moe_stack_set_spin_limit", _i, [_vp, _i]),
    ("moe_stack_set_trace", _i, [_vp, _vp, _sz]),
]


def library_path() -> str:
    return _build.LIB


def load() -> C.CDLL:
    """Load (building first if missing or stale) and declare the library."""
    global _L
    if _L is None:
        path = _build.build()
        if not os.path.exists(path):
            raise ImportError(f"CUDA library not found: {path}")
        lib = C.CDLL(path)
        for name, res, args in SIGNATURES:
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _L = lib
    return _L


class MoEError(RuntimeError):
    def __init__(self, call: str, code: int):
        self.code = code
        msg = load().moe_status_string(code).decode()
        super().__init__(f"{call} failed: {msg} ({code})")


def check(call: str, code: int) -> None:
    if code != MOE_OK:
        raise MoEError(call, code)
