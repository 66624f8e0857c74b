"""ctypes declarations of libwaits.so (include/waits.h), nothing else.

Loading never falls back to anything: a missing or unloadable library raises
``WaitsLibraryError``.
"""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwaits.so")

WAITS_OK = 0
STATUS_NAMES = {0: "WAITS_OK", 1: "WAITS_ERR_ARG", 2: "WAITS_ERR_SHAPE",
                3: "WAITS_ERR_UNSUPPORTED", 4: "WAITS_ERR_WORKSPACE",
                5: "WAITS_ERR_CUDA", 6: "WAITS_ERR_TIMEOUT",
                7: "WAITS_ERR_DEVICE"}
DEV_TIMEOUT, DEV_BAD_SEQLENS, DEV_PLAN_OVERFLOW, DEV_BAD_INDEX, DEV_BAD_CURVE = 1, 2, 4, 8, 16


class WaitsLibraryError(RuntimeError):
    pass


class WaitsError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("nseq", ctypes.c_int32), ("total_tokens", ctypes.c_int32),
                ("max_seqlen", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("cu_seqlens", ctypes.c_void_p)]


class DeviceBuffers(ctypes.Structure):
    _fields_ = [("Q", ctypes.c_void_p), ("K", ctypes.c_void_p),
                ("V", ctypes.c_void_p), ("scores", ctypes.c_void_p),
                ("idx", ctypes.c_void_p), ("kept_len", ctypes.c_void_p),
                ("K_out", ctypes.c_void_p), ("V_out", ctypes.c_void_p),
                ("cu_seqlens", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_PSHAPE = ctypes.POINTER(Shape)

# name -> (restype, argtypes); mirrors include/waits.h
SIGNATURES = {
    "waits_abi_version": (_I, []),
    "waits_strerror": (ctypes.c_char_p, [_I]),
    "waits_last_error": (ctypes.c_char_p, []),
    "waits_workspace_size": (_I, [_PSHAPE, ctypes.POINTER(_SZ)]),
    "waits_score": (_I, [_PSHAPE, _P, _P, _F, _I, _P, _P, _SZ, _P]),
    "waits_score_with_lse": (_I, [_PSHAPE, _P, _P, _P, _F, _I, _P, _P, _SZ, _P]),
    "waits_score_routed": (_I, [_PSHAPE, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "waits_compress_heads": (_I, [_PSHAPE, _I, _I, _P, _P, _P, _F, _I, _I, _I, _P, _P, _P,
                                  _P, _P, _P, _SZ, _P]),
    "waits_compress_routed": (_I, [_PSHAPE, _P, _P, _P, _P, _P, _I, _I, _P, _P, _P, _P, _P,
                                   _P, _SZ, _P]),
    "waits_select": (_I, [_PSHAPE, _P, _I, _I, _P, _P, _P, _SZ, _P]),
    "waits_compact": (_I, [_PSHAPE, _P, _P, _P, _P, _I, _P, _P, _P, _SZ, _P]),
    "waits_compress": (_I, [_PSHAPE, _P, _P, _P, _F, _I, _I, _I, _P, _P, _P,
                            _P, _P, _P, _SZ, _P]),
    "waits_compress_host": (_I, [_PSHAPE, _P, _P, _P, _P, _F, _I, _I, _I, _P,
                                 _P, _P, _P, ctypes.POINTER(DeviceBuffers), _P,
                                 _SZ, _P, ctypes.POINTER(_SZ),
                                 ctypes.POINTER(_SZ)]),
    "waits_read_device_status": (_I, [_P, _SZ, _P,
                                      ctypes.POINTER(ctypes.c_uint32)]),
    "waits_score_static": (_I, [_PSHAPE, _P, _P, _F, _I, _P, _P]),
    "waits_read_static_status": (_I, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "waits_test_exp2_poly": (_I, [_P, _P, ctypes.c_int64, _P]),
    "waits_decode_workspace_size": (_I, [_I, _I, _I, _I, ctypes.POINTER(_SZ)]),
    "waits_decode_attention": (_I, [_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "waits_score_kernels": (_I, [_PSHAPE, _F, _I, ctypes.POINTER(ctypes.c_int32)]),
    "waits_select_compact": (_I, [_PSHAPE, _P, _P, _P, _I, _I, _P, _P, _P, _P, _P, _SZ, _P]),
}

STATIC_WORKSPACE_BYTES = 32 << 20   # WAITS_STATIC_WORKSPACE_BYTES

_lib = None


def load(path: str = LIB_PATH):
    """Load libwaits.so (once) and declare every entry point."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise WaitsLibraryError(
            f"{path} is missing: build it with "
            "`python -m prefill_eviction_scoring_b200.build` (nvcc, sm_100a)")
    try:
        lib = ctypes.CDLL(path)
    except OSError as exc:
        raise WaitsLibraryError(f"cannot load {path}: {exc}") from exc
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(fn: str, status: int):
    if status != WAITS_OK:
        lib = load()
        msg = lib.waits_strerror(status).decode()
        if status == 5:
            msg += " [" + lib.waits_last_error().decode() + "]"
        raise WaitsError(fn, status, msg)
