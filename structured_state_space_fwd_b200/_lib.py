"""ctypes loader for libssd.so and the C types of include/ssd.h."""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
# SSD_LIBRARY selects another in-tree build of the library to load (the tests use
# it for libssd_testhooks.so); by default the shipped libssd.so
lib_path = os.environ.get("SSD_LIBRARY") or os.path.join(PKG, "libssd.so")

SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED, SSD_ERR_CUDA, SSD_ERR_TIMEOUT = range(5)
SSD_F32, SSD_BF16 = 0, 1


class ShapeT(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("nheads", ctypes.c_int64), ("headdim", ctypes.c_int64),
                ("ngroups", ctypes.c_int64), ("dstate", ctypes.c_int64),
                ("chunk_size", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class SSDError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = f"{where}: {status_string(status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


_lib = None
_lock = threading.Lock()

_VP = ctypes.c_void_p
_SIGS = {
    "ssd_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "ssd_last_error_detail": ([], ctypes.c_char_p),
    "ssd_version": ([], ctypes.c_int),
    "ssd_fwd_plan": ([ctypes.POINTER(ShapeT), ctypes.POINTER(ctypes.c_char_p),
                      ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
    "ssd_fwd_workspace_size": ([ctypes.POINTER(ShapeT), ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
    "ssd_fwd": ([ctypes.POINTER(ShapeT)] + [_VP] * 10 + [ctypes.c_size_t, _VP], ctypes.c_int),
    "ssd_fwd_host_workspace_size": ([ctypes.POINTER(ShapeT), ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
    "ssd_fwd_host": ([ctypes.POINTER(ShapeT)] + [_VP] * 10 + [ctypes.c_size_t, _VP], ctypes.c_int),
    "ssd_fwd_no_alloc": ([ctypes.POINTER(ShapeT)] + [_VP] * 10, ctypes.c_int),
    "ssd_fwd_no_alloc_check": ([ctypes.POINTER(ShapeT), _VP], ctypes.c_int),
    "ssd_fwd_check": ([ctypes.POINTER(ShapeT), _VP, ctypes.c_size_t, _VP], ctypes.c_int),
    "ssd_fwd_varlen_workspace_size": ([ctypes.POINTER(ShapeT), ctypes.c_int64,
                                       ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
    "ssd_fwd_varlen": ([ctypes.POINTER(ShapeT)] + [_VP] * 7 + [ctypes.c_int64] + [_VP] * 4
                       + [ctypes.c_size_t, _VP], ctypes.c_int),
    "ssd_fwd_varlen_check": ([ctypes.POINTER(ShapeT), ctypes.c_int64, _VP, ctypes.c_size_t, _VP],
                             ctypes.c_int),
    "ssd_fwd_gated_workspace_size": ([ctypes.POINTER(ShapeT), ctypes.c_int64, ctypes.c_int,
                                      ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
    "ssd_fwd_gated": ([ctypes.POINTER(ShapeT)] + [_VP] * 9 + [ctypes.c_int64, ctypes.c_float, ctypes.c_int]
                      + [_VP] * 3 + [ctypes.c_size_t, _VP], ctypes.c_int),
    "ssd_step": ([ctypes.POINTER(ShapeT)] + [_VP] * 9, ctypes.c_int),
    "ssd_cp_record_floats": ([ctypes.POINTER(ShapeT), ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
    "ssd_cp_workspace_size": ([ctypes.POINTER(ShapeT), ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
    "ssd_cp_begin": ([ctypes.POINTER(ShapeT)] + [_VP] * 7 + [ctypes.c_size_t, _VP], ctypes.c_int),
    "ssd_cp_end": ([ctypes.POINTER(ShapeT), ctypes.c_int, ctypes.c_int] + [_VP] * 10
                   + [ctypes.c_size_t, _VP], ctypes.c_int),
    "ssd_gated_rmsnorm": ([ctypes.POINTER(ShapeT), _VP, _VP, _VP, ctypes.c_int64, ctypes.c_float,
                           _VP, _VP], ctypes.c_int),
    "ssd_chunk_cumsum": ([ctypes.POINTER(ShapeT), _VP, _VP, _VP, _VP], ctypes.c_int),
    "ssd_chunk_state": ([ctypes.POINTER(ShapeT)] + [_VP] * 6, ctypes.c_int),
    "ssd_state_passing": ([ctypes.POINTER(ShapeT)] + [_VP] * 6, ctypes.c_int),
    "ssd_chunk_scan": ([ctypes.POINTER(ShapeT)] + [_VP] * 9, ctypes.c_int),
}


def lib():
    """Load libssd.so once; raise if it is missing (no fallback exists)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(lib_path):
                raise ImportError(f"libssd.so not built at {lib_path}; run "
                                  "`python -m structured_state_space_fwd_b200.build`")
            L = ctypes.CDLL(lib_path)
            for name, (args, res) in _SIGS.items():
                f = getattr(L, name)
                f.argtypes = args
                f.restype = res
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().ssd_status_string(int(status)).decode()


def check(status: int, where: str):
    if status != SSD_OK:
        detail = lib().ssd_last_error_detail().decode()
        raise SSDError(status, where, detail)
