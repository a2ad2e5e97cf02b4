"""ctypes loader for libkata.so (the C ABI declared in include/kata.h).

The shared library is built in-tree by ``kernelized_linear_attention_kata_b200.build``.
There is no fallback: if the library is missing or does not load, every entry
point raises.
"""

from __future__ import annotations

import ctypes
import os

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libkata.so")

# Enum values of include/kata.h
KATA_OK = 0
KATA_ERR_INVALID_ARGUMENT = 1
KATA_ERR_UNSUPPORTED = 2
KATA_ERR_WORKSPACE = 3
KATA_ERR_CUDA = 4
KATA_ERR_NONPOSITIVE_NORMALISER = 5
KATA_ERR_DEVICE_TIMEOUT = 6

KATA_PATH_NONE = 0
KATA_PATH_TENSOR_CORE_PSD = 1
KATA_PATH_TENSOR_CORE_FIRST_ORDER = 2
KATA_PATH_CUDA_CORE = 3
KATA_PATH_TENSOR_CORE_MULTI_FACTOR = 4
PATH_NAMES = {KATA_PATH_NONE: "none", KATA_PATH_TENSOR_CORE_PSD: "tensor_core_psd",
              KATA_PATH_TENSOR_CORE_FIRST_ORDER: "tensor_core_first_order",
              KATA_PATH_CUDA_CORE: "cuda_core",
              KATA_PATH_TENSOR_CORE_MULTI_FACTOR: "tensor_core_multi_factor"}

KATA_DTYPE_F32 = 0
KATA_DTYPE_BF16 = 1
KATA_FEATURE_PSD = 0
KATA_FEATURE_FIRST_ORDER = 1
KATA_FEATURE_MULTI_PSD2 = 2      # KATA-Mg, g = 2
KATA_FEATURE_SUMMED_PSD2 = 3     # KATA-Sigma-g, g = 2

class KataPlan(ctypes.Structure):
    """kata_plan_t"""
    _fields_ = [("path", ctypes.c_int), ("segments", ctypes.c_int),
                ("segment_tokens", ctypes.c_int), ("chunk_tokens", ctypes.c_int)]


# Every symbol the header declares, with (restype, argtypes).
_vp, _cvp, _i, _sz, _fp = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
_FWD = [_cvp, _cvp, _cvp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _fp, _fp, _vp, _sz, _vp]
SIGNATURES = {
    "kata_version": (ctypes.c_int, []),
    "kata_status_string": (ctypes.c_char_p, [_i]),
    "kata_state_dim": (ctypes.c_size_t, [_i, _i]),
    "kata_fwd_chunked_workspace_bytes": (ctypes.c_size_t, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "kata_fwd_chunked_plan": (ctypes.c_int, [_i, _i, _i, _i, _i, _i, _i, _i, _i,
                                             ctypes.POINTER(KataPlan)]),
    "kata_fwd_chunked": (ctypes.c_int, _FWD),
    "kata_fwd_chunked_sequential": (ctypes.c_int, _FWD),
    "kata_fwd_chunked_noalloc": (ctypes.c_int, [_cvp, _cvp, _cvp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                                                _fp, _fp, _vp]),
    "kata_fwd_chunked_from_state": (ctypes.c_int, [_cvp, _cvp, _cvp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                                   _i, _fp, _fp, _fp, _fp, _vp, _sz, _vp]),
    "kata_chunked_state": (ctypes.c_int, [_cvp, _cvp, _i, _i, _i, _i, _i, _i, _i, _i, _fp, _fp, _vp,
                                          _sz, _vp]),
    "kata_fwd_quadratic": (ctypes.c_int, [_cvp, _cvp, _cvp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "kata_decode_step": (ctypes.c_int, [_cvp, _cvp, _cvp, _fp, _fp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "kata_bwd_chunked_workspace_bytes": (ctypes.c_size_t, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "kata_bwd_chunked": (ctypes.c_int, [_cvp, _cvp, _cvp, _cvp, _vp, _vp, _vp, _i, _i, _i, _i,
                                        _i, _i, _i, _i, _vp, _sz, _vp]),
    "kata_fwd_delta": (ctypes.c_int, [_cvp, _cvp, _cvp, _fp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                      _fp, _fp, _vp, _sz, _vp]),
    "kata_workspace_status": (ctypes.c_int, [_cvp, _vp]),
    "kata_selftest_device_timeout": (ctypes.c_int, [_vp, _sz, _vp]),
    "kata_profile_enable": (ctypes.c_int, [_i]),
    "kata_profile_count": (ctypes.c_int, []),
    "kata_profile_get": (ctypes.c_int, [_i, ctypes.POINTER(ctypes.c_char_p),
                                        ctypes.POINTER(ctypes.c_longlong),
                                        ctypes.POINTER(ctypes.c_double)]),
}

_lib = None


class KataError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        name = lib().kata_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{fn} returned {name} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it is missing (no CPU fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"KATA CUDA library not built: {LIB_PATH} is missing. "
                "Run `python -m kernelized_linear_attention_kata_b200.build`.")
        handle = ctypes.CDLL(LIB_PATH, mode=ctypes.RTLD_LOCAL)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def check(fn: str, status: int) -> None:
    if status != KATA_OK:
        raise KataError(fn, status)
