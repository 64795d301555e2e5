"""ctypes loader for libnvfp4.so (the C ABI declared in include/nvfp4.h).

The library must have been built (``nvfp4_w4a4_gemm_quantize_b200.build``);
a missing library raises at first use -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnvfp4.so")

_lock = threading.Lock()
_LIB = None

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_status = ctypes.c_int

STATUS = {
    0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_UNSUPPORTED_SHAPE",
    3: "NVFP4_ERR_MISALIGNED", 4: "NVFP4_ERR_UNSUPPORTED_DEVICE", 5: "NVFP4_ERR_CUDA",
    6: "NVFP4_ERR_TIMEOUT", 7: "NVFP4_ERR_WORKSPACE", 8: "NVFP4_ERR_NONFINITE",
}

class NVFP4GemmProblem(ctypes.Structure):
    """nvfp4_gemm_problem (include/nvfp4.h): one product of a grouped call."""
    _fields_ = [("a_codes", _p), ("a_sf", _p), ("a_scale", _p),
                ("b_codes", _p), ("b_sf", _p), ("b_scale", _p),
                ("M", _i64), ("N", _i64), ("K", _i64),
                ("y", _p), ("y_codes", _p), ("y_sf", _p), ("y_scale", _p), ("y_amax", _p), ("act", _int)]


MAX_GROUP = 8

# every symbol include/nvfp4.h declares, with (restype, argtypes)
SIGNATURES = {
    "nvfp4_sf_bytes": (ctypes.c_size_t, [_i64, _i64]),
    "nvfp4_quantize_workspace_bytes": (ctypes.c_size_t, [_i64, _i64]),
    "nvfp4_quantize": (_status, [_p, _i64, _i64, _i64, _p, _p, _p, ctypes.c_uint, _p, ctypes.c_size_t, _p, _p]),
    "nvfp4_quantize_noalloc": (_status, [_p, _i64, _i64, _i64, _p, _p, _p, ctypes.c_uint, _p, _p]),
    "nvfp4_layernorm_quantize": (_status, [_p, _i64, _i64, _i64, _p, _p, _i64, ctypes.c_double, _p, _p, _p,
                                           ctypes.c_uint, _p, ctypes.c_size_t, _p, _p]),
    "nvfp4_dequantize": (_status, [_p, _p, _p, _i64, _i64, _p, _int, _p]),
    "nvfp4_quantize_block": (_status, [_p, _i64, _i64, _i64, _int, _p, _p, _p, ctypes.c_uint, _p, ctypes.c_size_t,
                                       _p, _p]),
    "nvfp4_block_size_errors": (_status, [_p, _i64, _i64, _i64, _p, _p, _p]),
    "nvfp4_select_block_size": (_int, [_p, ctypes.c_double]),
    "nvfp4_fake_quantize": (_status, [_p, _i64, _i64, _i64, _p, _int, _p, _p, ctypes.c_uint, _p, ctypes.c_size_t,
                                      _p, _p]),
    "nvfp4_ste_backward": (_status, [_p, _p, _i64, _i64, _int, _p, _p]),
    "nvfp4_gemm_w4a4": (_status, [_p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _p, _int, _p, _p, _p, _p, _int, _p,
                                  _p]),
    "nvfp4_gemm_w4a4_grouped": (_status, [_p, _int, _int, _p, _p]),
    "nvfp4_gemm_w4a16": (_status, [_p, _p, _p, _p, _i64, _i64, _i64, _p, _int, _p, _p]),
    "nvfp4_attention": (_status, [_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _p,
                                  ctypes.c_size_t, _p, _p]),
    "nvfp4_attention_workspace_bytes": (ctypes.c_size_t, [_i64, _i64, _i64]),
    "nvfp4_mx_sf_bytes": (ctypes.c_size_t, [_i64, _i64]),
    "nvfp4_mx_quantize": (_status, [_p, _i64, _i64, _i64, _p, _p, _p]),
    "nvfp4_mx_dequantize": (_status, [_p, _p, _i64, _i64, _p, _int, _p]),
    "nvfp4_mx_gemm": (_status, [_p, _p, _p, _p, _i64, _i64, _i64, _p, _int, _int, _p, _p]),
    "nvfp4_status_string": (ctypes.c_char_p, [_int]),
    "nvfp4_launch_count": (ctypes.c_uint64, []),
    "nvfp4_shutdown": (None, []),
    "nvfp4_debug_wait_timeout": (_status, [_p, _i64, _p]),
}


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = STATUS.get(status, str(status))
        msg = lib().nvfp4_status_string(status).decode() if _LIB is not None else name
        super().__init__(f"{where}: {name} ({msg})")


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        with _lock:
            if _LIB is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"{LIB_PATH} is missing: build it with "
                        "`python -m nvfp4_w4a4_gemm_quantize_b200.build` (nvcc, sm_100a)")
                L = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in SIGNATURES.items():
                    fn = getattr(L, name)
                    fn.restype = res
                    fn.argtypes = args
                _LIB = L
    return _LIB


def check(status: int, where: str) -> None:
    if status != 0:
        raise NVFP4Error(status, where)
