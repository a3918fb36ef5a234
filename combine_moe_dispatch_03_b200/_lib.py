"""ctypes loader for libmoe_dispatch.so (the C ABI in include/moe_dispatch.h).

The library is built in-tree by ``combine_moe_dispatch_03_b200.build``.  There
is no fallback: if the shared library is missing or fails to load, every entry
point raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_dispatch.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_CUDA = -2
MOE_ERR_SCRATCH = -3
NOALLOC_SCRATCH_BYTES = 4 << 20

ST_EXPERT_OOR = 1
ST_CAPACITY = 2
ST_ROW_OOR = 4
ST_COVERAGE = 8
ST_LAYOUT_MISMATCH = 16
ST_TIMEOUT = 32
STATUS_BITS = (ST_EXPERT_OOR, ST_CAPACITY, ST_ROW_OOR, ST_COVERAGE, ST_LAYOUT_MISMATCH, ST_TIMEOUT)

DTYPE_F32 = 0
DTYPE_BF16 = 1

MAX_K = 32
MAX_E = 1024
MAX_R = 64

# Exported symbols and their C signatures (restype, argtypes).
_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64
SIGNATURES = {
    "moe_layout_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "moe_worst_case_rows": (ctypes.c_int64, [_I, _I, _I, _I]),
    "moe_dispatch_layout": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_dispatch_layout_noalloc": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_permute": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _I, _L, _P, _P, _P, _P, _P]),
    "moe_dispatch": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _I, _L, _P,
                          _P, _P, _P, _P]),
    "moe_expert_scale": (_I, [_P, _L, _P, _P, _I, _I, _P, _P, _P, _P]),
    "moe_combine_weighted": (_I, [_P, _L, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "moe_combine_backward": (_I, [_P, _P, _L, _P, _P, _P, _I, _I, _I, _I, _P, _I, _I, _P, _P, _P,
                                  _P]),
    "moe_permute_payload": (_I, [_P, _L, _P, _L, _P, _I, _I, _I, _P, _P, _I, _L, _P, _P, _P, _P,
                                 _P, _P]),
    "moe_combine_weighted_f32": (_I, [_P, _L, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "moe_combine_backward_f32": (_I, [_P, _P, _L, _P, _P, _P, _I, _I, _I, _I, _P, _I, _I, _P, _P,
                                      _P, _P]),
    "moe_scatter_flat_index": (_I, [_P, _L, _I, _I, _P, _P, _P]),
    "moe_segment_labels": (_I, [_P, _I, _I, _L, _P, _P, _P]),
    "moe_rank_bases": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "moe_permute_to_ranks": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _L, _I, _P, _P, _I,
                                  _P, _P, _P]),
    "moe_combine_from_ranks": (_I, [_P, _P, _I, _I, _L, _P, _P, _I, _P, _I, _I, _I, _I, _P, _P,
                                    _P]),
    "moe_strerror": (ctypes.c_char_p, [_I]),
    "moe_status_bit_name": (ctypes.c_char_p, [_I]),
    "moe_last_cuda_error": (ctypes.c_char_p, []),
    "moe_version": (ctypes.c_char_p, []),
}

_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load the shared library once; raise if it is not there."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m combine_moe_dispatch_03_b200.build`"
                " (there is no CPU or Python fallback)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
        return handle


def check_rc(rc: int, what: str) -> None:
    if rc != MOE_OK:
        msg = lib().moe_strerror(rc).decode()
        if rc == MOE_ERR_CUDA:
            msg += f": {lib().moe_last_cuda_error().decode()}"
        raise RuntimeError(f"{what} failed: {msg} (code {rc})")


def decode_status(bits: int) -> list[str]:
    return [lib().moe_status_bit_name(b).decode() for b in STATUS_BITS if bits & b]
