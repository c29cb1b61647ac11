"""ctypes binding of libpisa_b200.so (include/pisa.h). Argument marshalling
only: every step of the path runs in the library's CUDA kernels.

Loading fails loudly when the library is missing; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpisa_b200.so")

PISA_OK = 0
STATUS_NAMES = {
    0: "PISA_OK", 1: "PISA_ERR_INVALID_ARGUMENT", 2: "PISA_ERR_UNSUPPORTED", 3: "PISA_ERR_WORKSPACE",
    4: "PISA_ERR_CAPACITY", 5: "PISA_ERR_CUDA", 6: "PISA_ERR_DEVICE",
}
DTYPE_F32 = 0
DTYPE_BF16 = 1

# Every symbol include/pisa.h declares, with (restype, argtypes).
_p = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64


class Config(ctypes.Structure):
    """Mirror of pisa_config."""
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "N", "H_q", "H_kv", "d", "C", "g", "K", "q_tile", "causal",
                                               "dtype")] + [("scale", ctypes.c_float)]


class QuerySpan(ctypes.Structure):
    """Mirror of pisa_query_span."""
    _fields_ = [("q0", ctypes.c_int32), ("n_q", ctypes.c_int32)]


class DecodeConfig(ctypes.Structure):
    """Mirror of pisa_decode_config."""
    _fields_ = [(n, ctypes.c_int32) for n in ("S", "cap", "H_q", "H_kv", "d", "C", "g", "K", "dtype")] + [
        ("scale", ctypes.c_float)]


_PC = ctypes.POINTER(Config)
_PS = ctypes.POINTER(QuerySpan)
_PD = ctypes.POINTER(DecodeConfig)

SIGNATURES = {
    "pisa_status_string": (ctypes.c_char_p, [_i32]),
    "pisa_version": (_i32, []),
    "pisa_launch_count": (ctypes.c_uint64, []),
    "pisa_device_faults": (ctypes.c_uint64, []),
    "pisa_timing_start": (_i32, []),
    "pisa_timing_stop": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                                        ctypes.POINTER(ctypes.c_int)]),
    "pisa_pyramid_geometry": (_i32, [_i64, _i32, _i32, ctypes.POINTER(_i32), _p]),
    "pisa_pyramid_rows": (_i64, [_i64, _i32]),
    "pisa_build_pyramid": (_i32, [_PC, _p, _p, _p]),
    "pisa_select_workspace_bytes": (ctypes.c_size_t, [_PC]),
    "pisa_select": (_i32, [_PC, _p, _p, _p, _p, _p, _p, ctypes.c_size_t, _p]),
    "pisa_select_flat_workspace_bytes": (ctypes.c_size_t, [_PC]),
    "pisa_select_flat": (_i32, [_PC, _p, _p, _p, _p, ctypes.c_size_t, _p]),
    "pisa_select_exact": (_i32, [_PC, _p, _p, _p, _p]),
    "pisa_attn_bwd_workspace_bytes": (ctypes.c_size_t, [_PC]),
    "pisa_sparse_attn_bwd": (_i32, [_PC, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, ctypes.c_size_t, _p]),
    "pisa_attn_fwd_workspace_bytes": (ctypes.c_size_t, [_PC]),
    "pisa_sparse_attn_fwd": (_i32, [_PC, _p, _p, _p, _p, _p, _p, _p, ctypes.c_size_t, _p]),
    "pisa_select_noalloc": (_i32, [_PC, _p, _p, _p, _p, _p, _p]),
    "pisa_select_span_workspace_bytes": (ctypes.c_size_t, [_PC, _PS]),
    "pisa_select_span": (_i32, [_PC, _PS, _p, _p, _p, _p, _p, _p, ctypes.c_size_t, _p]),
    "pisa_attn_fwd_span_workspace_bytes": (ctypes.c_size_t, [_PC, _PS]),
    "pisa_sparse_attn_fwd_span": (_i32, [_PC, _PS, _p, _p, _p, _p, _p, _p, _p, ctypes.c_size_t, _p]),
    "pisa_decode_pyramid_rows": (_i64, [_PD]),
    "pisa_decode_workspace_bytes": (_i64, [_PD]),
    "pisa_decode_init": (_i32, [_PD, _p, _p, _p, _p]),
    "pisa_decode_append": (_i32, [_PD, _p, _p, _p, _p, _p, _p, _p, _p]),
    "pisa_decode_select": (_i32, [_PD, _p, _p, _p, _p, _p, _p]),
    "pisa_decode_attn": (_i32, [_PD, _p, _p, _p, _p, _p, _p, _p, _p, _p]),
    "pisa_decode_step": (_i32, [_PD, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p]),
    "pisa_decode_init_paged": (_i32, [_PD, _p, _p, ctypes.c_int, _p, _p, _p]),
    "pisa_decode_step_paged": (_i32, [_PD, _p, _p, _p, _p, _p, _p, ctypes.c_int, _p, _p, _p, _p, _p, _p, _p, _p]),
}

_lock = threading.Lock()
_lib = None


class PisaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: run `python -m hierarchical_top_block_mean_b200.build` "
                                  "(the CUDA library is required; there is no CPU fallback)")
            h = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(h, name)
                f.restype = res
                f.argtypes = args
            _lib = h
    return _lib


def call(name: str, *args) -> None:
    """Calls an entry point that returns pisa_status; raises PisaError unless PISA_OK."""
    st = getattr(lib(), name)(*args)
    if st != PISA_OK:
        raise PisaError(name, st)
