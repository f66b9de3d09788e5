"""ctypes view of libfa_b200.so (the C ABI declared in include/fa.h).

Loading fails loudly if the library has not been built; there is no
fallback implementation anywhere in the package.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libfa_b200.so")

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_CUDA = 3
FA_ERR_DEVICE_TIMEOUT = 4
FA_BF16 = 0
FA_F32 = 1
# Backward phase bits (include/fa.h FA_BWD_PHASE_*) and the two whole passes.
BWD_PREPROCESS = 0x01
BWD_DKDV = 0x02
BWD_DQ = 0x04
BWD_FUSED_KERNEL = 0x08
BWD_DQ_CONVERT = 0x10
BWD_SPLIT = 0x07
BWD_FUSED = 0x19

c_void_p = ctypes.c_void_p
c_int = ctypes.c_int
c_ll = ctypes.c_longlong
c_float = ctypes.c_float
c_size_t = ctypes.c_size_t

# name -> (restype, argtypes), one entry per function in include/fa.h
SIGNATURES = {
    "fa_fwd": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                       c_int, c_int, c_int, c_int, c_float, c_void_p, c_int, c_ll, c_void_p]),
    "fa_bwd_workspace_size": (c_size_t, [c_ll, c_int, c_int, c_int]),
    "fa_bwd_phases_workspace_size": (c_size_t, [ctypes.c_uint, c_ll, c_int, c_int, c_int]),
    "fa_bwd": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                       c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                       c_float, c_void_p, c_int, c_ll, c_void_p, c_size_t, c_void_p]),
    "fa_bwd_phases": (c_int, [ctypes.c_uint, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                              c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
                              c_int, c_int, c_int, c_float, c_void_p, c_int, c_ll, c_void_p,
                              c_size_t, c_void_p]),
    "fa_bwd_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                               c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
                               c_int, c_int, c_float, c_void_p, c_int, c_ll, c_void_p]),
    "fa_get_error_string": (ctypes.c_char_p, [c_int]),
    "fa_last_cuda_error_string": (ctypes.c_char_p, []),
    "fa_check_device_error": (c_int, [c_void_p, ctypes.POINTER(ctypes.c_uint)]),
    "fa_set_wait_budget": (None, [c_ll]),
    "fa_selftest_wait_timeout": (c_int, [c_ll, c_void_p]),
    "fa_selftest_exp2": (c_int, [c_void_p, c_void_p, c_ll, c_void_p]),
    "fa_decode_num_splits": (c_int, [c_int, c_int, c_int, c_int]),
    "fa_decode_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int, c_int]),
    "fa_decode": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                          c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_ll, c_int, c_int,
                          c_float, c_int, c_void_p, c_size_t, c_void_p]),
    "fa_fp8_quantize": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
                                c_void_p]),
    "fa_fwd_fp8": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                           c_int, c_int, c_int, c_int, c_int, c_int, c_float, c_void_p]),
    "fa_version": (c_int, []),
    "fa_debug_build": (c_int, []),
    "fa_debug_set_trace": (c_int, [c_void_p, c_size_t, c_int]),
}
DEBUG_TRACE_BYTES = 32 * 1024 * 8
DEBUG_LIB_PATH = os.path.join(PKG, "libfa_b200_debug.so")

_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = lib().fa_get_error_string(status).decode() if _lib is not None else str(status)
        if status == FA_ERR_CUDA and _lib is not None:
            msg += f" ({lib().fa_last_cuda_error_string().decode()})"
        super().__init__(f"{what}: {msg}")


def _load(path: str) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m exact_io_aware_tmem_b200.build`"
            " (the package has no non-CUDA fallback)")
    handle = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(handle, name)
        fn.restype = res
        fn.argtypes = args
    return handle


def lib() -> ctypes.CDLL:
    """The loaded library (loaded once)."""
    global _lib
    if _lib is None:
        _lib = _load(LIB_PATH)
    return _lib


_debug_lib = None


def debug_lib() -> ctypes.CDLL:
    """The debug build (index checks, event stamps); loaded once, on request."""
    global _debug_lib
    if _debug_lib is None:
        _debug_lib = _load(DEBUG_LIB_PATH)
    return _debug_lib


def check(status: int, what: str) -> None:
    if status != FA_OK:
        raise FAError(status, what)
