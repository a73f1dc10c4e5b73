"""ctypes loader for libmuon_b200.so and the C-ABI declarations of include/muon_b200.h.

The library is built in-tree (``python -m muon_polar_orthogonalized_b200.build``)
and loaded from this package directory.  There is no fallback: if the library
is missing or cannot be loaded, every entry point raises.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import (POINTER, c_char_p, c_double, c_float, c_int, c_int32, c_int64, c_size_t,
                    c_uint32, c_void_p)

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libmuon_b200.so")

# status codes (muon_status)
MUON_OK = 0
MUON_ERR_INVALID_ARG = 1
MUON_ERR_UNSUPPORTED = 2
MUON_ERR_WORKSPACE = 3
MUON_ERR_CUDA = 4
MUON_ERR_TIMEOUT = 5

# dtypes and flags
MUON_F32 = 0
MUON_BF16 = 1
MUON_NESTEROV = 1
MUON_CAUTIOUS_WD = 2
MUON_FP32_DEBUG = 4
MUON_UNFUSED_UPDATE = 8
MUON_TC_SINGLE_CTA = 16
MUON_NORMUON = 32
MUON_ROW_EQUILIBRATE = 64
MUON_TC_NARROW_TILES = 128
MUON_TC_WIDE_TILES = 256


class MuonGroup(ctypes.Structure):
    _fields_ = [("rows", c_int32), ("cols", c_int32), ("count", c_int32), ("first", c_int32),
                ("grad_dtype", c_int32), ("lr_scale", c_float)]


class AdamWGroup(ctypes.Structure):
    _fields_ = [("params", POINTER(c_void_p)), ("grads", POINTER(c_void_p)),
                ("exp_avg", POINTER(c_void_p)), ("exp_avg_sq", POINTER(c_void_p)),
                ("numel", POINTER(c_int64)), ("count", c_int32), ("grad_dtype", c_int32),
                ("lr", c_float), ("beta1", c_float), ("beta2", c_float), ("eps", c_float),
                ("wd", c_float)]


# name -> (restype, argtypes); every function include/muon_b200.h declares
SIGNATURES = {
    "muon_workspace_size": (c_size_t, [POINTER(MuonGroup), c_int, c_uint32]),
    "muon_workspace_min_size": (c_size_t, [POINTER(MuonGroup), c_int, c_uint32]),
    "muon_step": (c_int, [POINTER(c_void_p), POINTER(c_void_p), POINTER(c_void_p),
                          POINTER(MuonGroup), c_int, c_float, c_float, c_float, c_int,
                          POINTER(c_float), c_uint32, c_void_p, c_size_t, c_void_p]),
    "muon_step_noalloc": (c_int, [POINTER(c_void_p), POINTER(c_void_p), POINTER(c_void_p),
                                  POINTER(MuonGroup), c_int, c_float, c_float, c_float, c_int,
                                  POINTER(c_float), c_uint32, c_void_p]),
    "muon_noalloc_scratch": (c_int, [POINTER(c_void_p), POINTER(c_size_t)]),
    "muon_orthogonalize": (c_int, [POINTER(c_void_p), POINTER(c_void_p), POINTER(MuonGroup), c_int,
                                   c_int, POINTER(c_float), c_uint32, c_void_p, c_size_t, c_void_p]),
    "adamw_step": (c_int, [POINTER(AdamWGroup), c_int, c_int64, c_void_p]),
    "muon_step_replicated": (c_int, [POINTER(c_void_p), POINTER(c_void_p), POINTER(c_void_p),
                                     POINTER(MuonGroup), c_int, c_float, c_float, c_float, c_int,
                                     POINTER(c_float), c_uint32, c_void_p, c_size_t,
                                     POINTER(POINTER(c_void_p)), c_int, c_void_p]),
    "muon_reduce_mean": (c_int, [POINTER(c_void_p), POINTER(POINTER(c_void_p)), c_int, POINTER(c_int64),
                                 c_int, c_int32, c_void_p]),
    "muon_schedule_advance": (c_int, [c_void_p, c_int64, c_float, c_float, c_float, c_void_p]),
    "muon_schedule_advance_cosine": (c_int, [c_void_p, c_int64, c_int64, c_float, c_void_p]),
    "muon_step_scheduled": (c_int, [POINTER(c_void_p), POINTER(c_void_p), POINTER(c_void_p),
                                    POINTER(MuonGroup), c_int, c_float, c_float, c_float, c_int,
                                    POINTER(c_float), c_uint32, c_void_p, c_size_t, c_void_p,
                                    c_void_p]),
    "adamw_step_scheduled": (c_int, [POINTER(AdamWGroup), c_int, c_void_p, c_void_p]),
    "muon_query_status": (c_int, [c_void_p, c_void_p]),
    "adamw_query_status": (c_int, [c_void_p]),
    "muon_selftest_wait_timeout": (c_int, [c_void_p, ctypes.c_uint64, c_void_p]),
    "muon_status_string": (c_char_p, [c_int]),
    "muon_last_error": (c_char_p, []),
    "muon_profiler_enable": (c_int, [c_int]),
    "muon_profiler_reset": (None, []),
    "muon_profiler_read": (c_int, [POINTER(c_double), POINTER(c_int64), c_int]),
    "muon_kernel_kind_count": (c_int, []),
    "muon_kernel_kind_name": (c_char_p, [c_int]),
}

_lib = None


class MuonError(RuntimeError):
    def __init__(self, status: int, fn: str, detail: str):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)}: {detail}")


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it is missing: there is no CPU fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} not found: build it with `python -m muon_polar_orthogonalized_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(st: int) -> str:
    return lib().muon_status_string(st).decode()


def last_error() -> str:
    return lib().muon_last_error().decode()


def check(st: int, fn: str) -> None:
    if st != MUON_OK:
        raise MuonError(st, fn, last_error())
