"""ctypes declarations of libmoeact.so (include/moeact.h).  Argument
marshalling only; every computation happens in the library's kernels.

The library must have been built (``python -m moe_gated_activation_b200.build``
or ``__graft_entry__.build()``); loading fails loudly otherwise -- there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoeact.so")

OK, EINVAL, EALIGN, EUNSUPPORTED, ERANGE, ECUDA, EWORKSPACE = range(7)
ROWWISE, COLWISE = 1, 2
DEV_OK, DEV_NEGATIVE_SPLIT, DEV_SPLIT_SUM, DEV_BAD_OFFSETS, DEV_UNALIGNED_GROUPS = range(5)
SCALES_ROWMAJOR, SCALES_GEMM = 0, 1
DEVERR_FWD_WAIT, DEVERR_BWD_WAIT, DEVERR_TABLE_WAIT, DEVERR_TABLE_ADDR = 0x1, 0x2, 0x4, 0x8
DEVERR_WAIT_SELFTEST, DEVERR_FC2_WAIT = 0x10, 0x20
MAX_GROUPS = 2040


class MxOut(ctypes.Structure):
    _fields_ = [("row_codes", ctypes.c_void_p), ("row_scales", ctypes.c_void_p),
                ("col_codes", ctypes.c_void_p), ("col_scales", ctypes.c_void_p),
                ("scale_layout", ctypes.c_int32), ("noop_flag", ctypes.c_void_p)]


class MoeactError(RuntimeError):
    def __init__(self, status, func, detail):
        self.status = status
        super().__init__(f"{func}: {detail} (status {status})")


_lock = threading.Lock()
_lib = None

P = ctypes.c_void_p
I64 = ctypes.c_int64
I32 = ctypes.c_int32
I = ctypes.c_int
SZ = ctypes.c_size_t
F = ctypes.c_float

_SIGS = {
    "moeact_init": ([], I),
    "moeact_status_string": ([I], ctypes.c_char_p),
    "moeact_last_error": ([], ctypes.c_char_p),
    "splits_to_offsets": ([P, I32, I64, P, P, P, P], I),
    "scaled_swiglu_mxfp8_fwd": ([P, I64, P, I64, I64, I, I, I32, MxOut, P], I),
    "scaled_srelu_mxfp8_fwd": ([P, I64, P, I64, I64, I, MxOut, P], I),
    "grouped_scaled_swiglu_mxfp8_fwd": ([P, I64, P, I64, I64, I, I, I32, P, P, I32, P, MxOut, P],
                                        I),
    "grouped_scaled_srelu_mxfp8_fwd": ([P, I64, P, I64, I64, I, P, P, I32, P, MxOut, P], I),
    "scaled_act_mxfp8_bwd_workspace_size": ([I64, I64, I32], SZ),
    "scaled_swiglu_mxfp8_bwd": ([P, I64, P, I64, P, I64, I64, I, I32, P, P, MxOut, P, SZ, P], I),
    "scaled_srelu_mxfp8_bwd": ([P, I64, P, I64, P, I64, I64, I, P, P, MxOut, P, SZ, P], I),
    "grouped_scaled_swiglu_mxfp8_bwd": ([P, I64, P, I64, P, I64, I64, I, I32, P, P, I32, P, P, P,
                                         MxOut, P, SZ, P], I),
    "grouped_scaled_srelu_mxfp8_bwd": ([P, I64, P, I64, P, I64, I64, I, P, P, I32, P, P, P,
                                        MxOut, P, SZ, P], I),
    "moeact_sigmoid_dump": ([P, P], I),
    "moeact_init_clamped": ([F, F], I),
    "scaled_clamped_swiglu_mxfp8_fwd": ([P, I64, P, I64, I64, I, F, F, I32, MxOut, P], I),
    "grouped_scaled_clamped_swiglu_mxfp8_fwd": ([P, I64, P, I64, I64, I, F, F, I32, P, P, I32, P,
                                                 MxOut, P], I),
    "scaled_clamped_swiglu_mxfp8_bwd": ([P, I64, P, I64, P, I64, I64, I, F, F, I32, P, P, MxOut,
                                         P, SZ, P], I),
    "grouped_scaled_clamped_swiglu_mxfp8_bwd": ([P, I64, P, I64, P, I64, I64, I, F, F, I32, P, P,
                                                 I32, P, P, P, MxOut, P, SZ, P], I),
    "moeact_clamped_sigmoid_dump": ([F, F, P, P], I),
    "moeact_device_error": ([P], I),
    "moeact_wait_selftest": ([I, ctypes.c_uint32, P, P], I),
    "grouped_scaled_swiglu_mxfp8_fc2": ([P, I64, P, I64, I64, I, P, I32, P, P, P, I64, P, I64, P,
                                         P], I),
    "scaled_swiglu_mxfp8_bwd_noalloc": ([P, I64, P, I64, P, I64, I64, I, P, P, MxOut, P], I),
}


def lib():
    """The loaded library (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m moe_gated_activation_b200.build`"
                " (the CUDA path has no fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def check(status, func):
    if status != OK:
        detail = lib().moeact_last_error().decode() or lib().moeact_status_string(status).decode()
        raise MoeactError(status, func, detail)


def call(name, *args):
    st = getattr(lib(), name)(*args)
    check(st, name)
    return st
