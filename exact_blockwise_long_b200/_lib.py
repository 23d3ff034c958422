"""ctypes loader for libringattn.so (the C ABI in include/ringattn.h).

The library is built in-tree (``python -m exact_blockwise_long_b200.build``);
nothing here falls back to another implementation: if the shared library is
missing, every call raises.
"""

from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libringattn.so")
CHECKED_LIB_PATH = os.path.join(_HERE, "libringattn_checked.so")  # built with --checked

RA_BF16 = 0
RA_F32 = 1

STATUS = {
    0: "RA_OK", -1: "RA_ERR_ARG", -2: "RA_ERR_SHAPE", -3: "RA_ERR_DTYPE", -4: "RA_ERR_ALIGN",
    -5: "RA_ERR_UNSUPPORTED", -6: "RA_ERR_CUDA", -7: "RA_ERR_TIMEOUT", -8: "RA_ERR_WORKSPACE",
    -9: "RA_ERR_BOUNDS",
}

# name -> (restype, argtypes); the order mirrors include/ringattn.h
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t
SIGNATURES = {
    "ringattn_version": (_I, []),
    "ringattn_status_string": (ctypes.c_char_p, [_I]),
    "ringattn_kernel_plan": (ctypes.c_char_p, [_I, _I64, _I64, _I, _I]),
    "ringattn_fwd": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _I, _F, _P]),
    "ringattn_fwd_gqa": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _I, _F, _P]),
    "ringattn_bwd_gqa": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _I,
                              _F, _P, _SZ, _P]),
    "ringattn_fwd_step": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _I, _F, _I, _P]),
    "ringattn_merge": (_I, [_P, _P, _P, _P, _I64, _I64, _P]),
    "ringattn_bwd_workspace_size": (_SZ, [_I64, _I64, _I64, _I64]),
    "ringattn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _I, _F,
                          _P, _SZ, _P]),
    "ringattn_bwd_phase": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _I,
                                _F, _P, _SZ, _I, _P]),
    "ringattn_bwd_prepare_size": (_SZ, [_I64, _I64, _I64]),
    "ringattn_bwd_prepare": (_I, [_P, _P, _P, _P, _SZ, _I64, _I64, _I64, _I64, _I, _P]),
    "ringattn_bwd_pair": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _F, _I,
                               _P]),
    "ringattn_bwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _I,
                                  _F, _P]),
    "ringattn_step_host_size": (_SZ, [_I64, _I64, _I64, _I64]),
    "ringattn_step_host": (_I, [_P] * 10 + [_SZ, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _I, _F] + [_P] * 7),
    "ringattn_decode_workspace_size": (_SZ, [_I64, _I64, _I64, _I64, _I, _I]),
    "ringattn_decode": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _I, _I, _I, _F, _P, _SZ, _P]),
    "blockwise_ffn_workspace_size": (_SZ, [_I64, _I64, _I]),
    "blockwise_ffn": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I, _P, _SZ, _P]),
    "blockwise_ffn_bwd_workspace_size": (_SZ, [_I64, _I64, _I]),
    "blockwise_ffn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I, _P, _SZ, _P]),
    "blockwise_layer_saved_size": (_SZ, [_I64, _I64, _I64, _I64]),
    "blockwise_layer_fwd_workspace_size": (_SZ, [_I64, _I64]),
    "blockwise_layer_bwd_workspace_size": (_SZ, [_I64, _I64, _I64, _I64, _I64, _I64]),
    "blockwise_layer_fwd": (_I, [_P] * 12 + [_SZ, _I64, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _I, _F, _P, _SZ,
                                             _P, _P]),
    "blockwise_layer_bwd": (_I, [_P] * 11 + [_SZ] + [_P] * 11 + [_I64, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _I,
                                                                  _P, _SZ, _P, _P]),
    "ringattn_accumulate": (_I, [_P, _P, _I64, _I, _P]),
    "ringattn_cast": (_I, [_P, _P, _I64, _I, _P]),
    "ringattn_get_error": (_I, [_P]),
    "ringattn_selftest_timeout": (_I, [_I, _P]),
}

_lock = threading.Lock()
_lib = None


class RingAttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")


def load(path: str) -> ctypes.CDLL:
    """A handle on a build of the library at `path` with the ABI's signatures."""
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m exact_blockwise_long_b200.build` "
            "(there is no fallback implementation)")
    h = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(h, name)
        f.restype = res
        f.argtypes = args
    return h


def lib() -> ctypes.CDLL:
    """Load the shared library once; raise if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = load(LIB_PATH)
    return _lib


def call(name: str, *args) -> int:
    """Call an ABI entry point returning a status; raise on a negative one."""
    rc = getattr(lib(), name)(*args)
    if rc != 0:
        raise RingAttnError(name, rc)
    return rc
