"""ctypes declarations of the C ABI in include/spade.h.

Loading fails loudly when libspade.so is missing: there is no other
implementation of these entry points.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import c_float, c_int, c_int32, c_int64, c_size_t, c_void_p, POINTER

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspade.so")

SPADE_OK, SPADE_ERR_INVALID, SPADE_ERR_UNSUPPORTED, SPADE_ERR_CUDA, SPADE_ERR_TIMEOUT, SPADE_ERR_WORKSPACE = range(6)
SPADE_F32, SPADE_BF16 = 0, 1


class SpadeGeom(ctypes.Structure):
    _fields_ = [("T", c_int32), ("H", c_int32), ("W", c_int32),
                ("bt", c_int32), ("bh", c_int32), ("bw", c_int32)]


class SpadeHeadScheme(ctypes.Structure):
    _fields_ = [("scheme", c_int32), ("tau", c_float), ("dense", c_int32)]


# name -> (restype, argtypes), in the order of include/spade.h
SIGNATURES = {
    "spade_tile3d": (c_int, [c_void_p, c_void_p, SpadeGeom, c_int, c_int, c_int, c_void_p]),
    "spade_summarize": (c_int, [c_void_p, c_void_p, SpadeGeom, c_int, c_int, c_int, c_void_p]),
    "spade_summarize_qk": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, SpadeGeom, c_int, c_int, c_int,
                                   c_void_p]),
    "spade_estimate": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_void_p]),
    "spade_estimate_scores": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_void_p]),
    "spade_select": (c_int, [c_void_p, POINTER(c_float), c_void_p, c_void_p, c_int, c_int, c_void_p]),
    "spade_select_scores": (c_int, [c_void_p, POINTER(c_float), c_void_p, c_void_p, c_int, c_int, c_void_p]),
    "spade_attn_workspace_bytes": (c_size_t, [SpadeGeom, c_int, c_int, c_int]),
    "spade_block_sparse_attn": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                        SpadeGeom, c_int, c_int, c_int, c_int, c_void_p, c_size_t,
                                        c_void_p]),
    "spade_block_sparse_attn_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                                SpadeGeom, c_int, c_int, c_int, c_int, c_void_p]),
    "spade_grouped_workspace_bytes": (c_size_t, [POINTER(SpadeGeom), c_int, POINTER(SpadeHeadScheme),
                                                 c_int, c_int, c_int]),
    "spade_grouped_attn": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, POINTER(SpadeGeom), c_int,
                                   POINTER(SpadeHeadScheme), c_int, c_int, c_int, c_int, c_void_p,
                                   c_size_t, c_void_p]),
    "spade_grouped_attn_lists": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, POINTER(SpadeGeom), c_int,
                                         POINTER(SpadeHeadScheme), c_int, c_int, c_int, c_int, c_void_p,
                                         c_size_t, c_void_p]),
    "spade_grouped_head_lists": (c_int, [POINTER(SpadeGeom), c_int, POINTER(SpadeHeadScheme), c_int,
                                         c_int, c_int, c_int, POINTER(c_int64), POINTER(c_int64)]),
    "spade_summarize_mode": (c_int, [c_void_p, c_void_p, SpadeGeom, c_int, c_int, c_int, c_int, c_void_p]),
    "spade_grouped_attn_ex": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, POINTER(SpadeGeom), c_int,
                                      POINTER(SpadeHeadScheme), c_int, c_int, c_int, c_int, c_int, c_int,
                                      c_void_p, c_void_p, c_size_t, c_void_p]),
    "spade_select_window": (c_int, [c_void_p, POINTER(c_float), POINTER(ctypes.c_int), SpadeGeom, c_void_p,
                                    c_void_p, c_int, c_void_p]),
    "spade_copy_head_slice": (c_int, [c_void_p, c_void_p, c_int64, c_int, c_int, c_int, c_int, c_int, c_int,
                                      c_void_p]),
    "spade_sics_workspace_bytes": (c_size_t, [POINTER(SpadeGeom), c_int, c_int]),
    "spade_sics": (c_int, [c_void_p, c_void_p, POINTER(SpadeGeom), c_int, c_int, c_int, c_int, c_void_p, c_void_p,
                           c_void_p, c_size_t, c_void_p]),
    "spade_grouped_host_workspace_bytes": (c_size_t, [POINTER(SpadeGeom), c_int, POINTER(SpadeHeadScheme), c_int,
                                                      c_int, c_int, c_int, c_int]),
    "spade_grouped_attn_host": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, POINTER(SpadeGeom), c_int,
                                        POINTER(SpadeHeadScheme), c_int, c_int, c_int, c_int, c_int, c_void_p,
                                        c_size_t, c_void_p]),
    "spade_last_device_status": (c_int, [c_void_p]),
    "spade_status_string": (ctypes.c_char_p, [c_int]),
    "spade_last_error_message": (ctypes.c_char_p, []),
    "spade_version": (c_int, []),
    "spade_selftest_bounded_wait": (c_int, [c_int64, c_void_p]),
}

_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m input_adaptive_block_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class SpadeError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load()
        msg = lib.spade_status_string(status).decode()
        detail = lib.spade_last_error_message().decode()
        super().__init__(f"{where}: {msg} ({detail})")
        self.status = status


def check(status: int, where: str) -> None:
    if status != SPADE_OK:
        raise SpadeError(status, where)
