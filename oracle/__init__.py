"""CPU oracle for MoE token dispatch and combine -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
Python binding) never imports, links or executes anything here, and nothing
here imports the product.  The arithmetic lives in ``moe_oracle.c`` (plain
C, fp64 where floating point); this module only compiles it with gcc, loads
it with ctypes and marshals numpy arrays.  The checker is the plain,
single-threaded build.  ``use_openmp()`` switches to a second build of the
same source with ``-fopenmp`` (identical results: its pragmas only split
independent loop iterations), which the benchmark's multi-core CPU-baseline
leg times.

Every function cites the passage it follows in ``moe_oracle.c``.  Parity
status of each function (what pins it) is listed in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_LIB_OMP = os.path.join(_HERE, "libmoe_oracle_omp.so")
_lock = threading.Lock()
_libs: dict = {}
_variant = "plain"

# Status bits of the documented contract (this package's own copy).
EXPERT_OOR = 1
CAPACITY = 2
ROW_OOR = 4
COVERAGE = 8


def build(force: bool = False, openmp: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so next to it (gcc, -O2, no FMA
    contraction so every rounding is the one written in the source); with
    ``openmp``, the same source with -fopenmp into libmoe_oracle_omp.so."""
    out = _LIB_OMP if openmp else _LIB
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
           *(["-fopenmp"] if openmp else []), "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def use_openmp(on: bool = True) -> None:
    """Route every function of this module to the OpenMP build (on) or back
    to the plain single-threaded checker (off)."""
    global _variant
    _variant = "openmp" if on else "plain"


def threads() -> int:
    """Threads the current build's loops may use (1 for the plain build)."""
    return int(_load().oracle_threads())


def _load():
    with _lock:
        lib = _libs.get(_variant)
        if lib is not None:
            return lib
        lib = ctypes.CDLL(build(openmp=_variant == "openmp"))
        P = ctypes.c_void_p
        I = ctypes.c_int
        L = ctypes.c_int64
        lib.oracle_bf16_from_float.argtypes = [ctypes.c_float]
        lib.oracle_bf16_from_float.restype = ctypes.c_uint16
        lib.oracle_bf16_round_array.argtypes = [P, L, P]
        lib.oracle_bf16_round_array.restype = None
        lib.oracle_layout.argtypes = [P, I, I, I, I, I, P, P, P, P, P, P]
        lib.oracle_layout.restype = I
        lib.oracle_output_splits.argtypes = [P, I, I, I, I, P]
        lib.oracle_output_splits.restype = None
        lib.oracle_permute.argtypes = [P, P, I, I, I, I, P, I, L, P, P, P]
        lib.oracle_permute.restype = I
        lib.oracle_bruteforce_rows.argtypes = [P, I, I, I, P, P]
        lib.oracle_bruteforce_rows.restype = None
        lib.oracle_expert_scale.argtypes = [P, P, P, I, I, P, P]
        lib.oracle_expert_scale.restype = None
        lib.oracle_combine.argtypes = [P, L, P, P, I, I, I, P, P]
        lib.oracle_combine.restype = I
        lib.oracle_check_coverage.argtypes = [P, P, L, L]
        lib.oracle_check_coverage.restype = I
        lib.oracle_scatter_flat_index.argtypes = [P, L, L, P]
        lib.oracle_scatter_flat_index.restype = I
        lib.oracle_combine_backward.argtypes = [P, P, L, P, P, P, I, I, I, P, I, I, P, P]
        lib.oracle_combine_backward.restype = I
        lib.oracle_restore_activation_dtype.argtypes = [P, L, P, P, P, I, I, I, P, P]
        lib.oracle_restore_activation_dtype.restype = I
        lib.oracle_permute_payload.argtypes = [P, L, P, L, P, I, I, I, P, I, L, P, P, P, P]
        lib.oracle_permute_payload.restype = I
        lib.oracle_combine_f32.argtypes = [P, L, P, P, I, I, I, P, P]
        lib.oracle_combine_f32.restype = I
        lib.oracle_combine_backward_f32.argtypes = [P, P, L, P, P, P, I, I, I, P, I, I, P, P]
        lib.oracle_combine_backward_f32.restype = I
        lib.oracle_rank_bases.argtypes = [P, I, I, I, I, P, P, P, P]
        lib.oracle_rank_bases.restype = I
        lib.oracle_threads.argtypes = []
        lib.oracle_threads.restype = I
        _libs[_variant] = lib
        return lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ------------------------------------------------------------------ bf16 ---

def bf16_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 bit patterns (uint16), RNE."""
    x = _c(np.asarray(x, dtype=np.float32), np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_bf16_round_array(_p(x), x.size, _p(out))
    return out


def f32_from_bf16(h: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float32 exactly."""
    h = np.asarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- layout ---

def layout(topk_idx: np.ndarray, E: int, R: int, align: int) -> dict:
    """get_dispatch_layout + count matrix + padded offsets (see moe_oracle.c)."""
    topk_idx = _c(topk_idx, np.int64)
    T, K = topk_idx.shape
    El = E // R
    out = dict(
        tokens_per_expert=np.zeros(E, np.int32),
        counts=np.zeros((R, R, El), np.int32),
        splits=np.zeros((R, R), np.int32),
        tokens_per_rank=np.zeros((R, R), np.int32),
        is_token_in_rank=np.zeros((T, R), np.uint8),
        expert_offsets=np.zeros(E + 1, np.int32),
    )
    st = _load().oracle_layout(_p(topk_idx), T, K, E, R, align, _p(out["tokens_per_expert"]),
                               _p(out["counts"]), _p(out["splits"]), _p(out["tokens_per_rank"]),
                               _p(out["is_token_in_rank"]), _p(out["expert_offsets"]))
    out["status"] = st
    return out


def output_splits(topk_idx: np.ndarray, E: int, R: int) -> np.ndarray:
    """[R_dest, R_src] assignments sent from source block s to rank r, counted
    directly (independent of the count matrix)."""
    topk_idx = _c(topk_idx, np.int64)
    T, K = topk_idx.shape
    out = np.zeros((R, R), np.int32)
    _load().oracle_output_splits(_p(topk_idx), T, K, E, R, _p(out))
    return out


def rank_bases(all_counts: np.ndarray, rank: int, align: int) -> dict:
    """Row bases of the direct expert-parallel dispatch from the per-expert
    counts of every source rank ([R, E]): dest_base [E], own_offsets
    [E/R + 1], own_counts [E/R], max_rows (see moe_oracle.c)."""
    all_counts = _c(all_counts, np.int32)
    R, E = all_counts.shape
    El = E // R
    out = dict(dest_base=np.zeros(E, np.int32), own_offsets=np.zeros(El + 1, np.int32),
               own_counts=np.zeros(El, np.int32))
    mx = np.zeros(1, np.int32)
    st = _load().oracle_rank_bases(_p(all_counts), R, E, rank, align, _p(out["dest_base"]),
                                   _p(out["own_offsets"]), _p(out["own_counts"]), _p(mx))
    out["max_rows"] = int(mx[0])
    out["status"] = st
    return out


# --------------------------------------------------------------- permute ---

def permute(x_bf16: np.ndarray, topk_idx: np.ndarray, E: int, expert_offsets: np.ndarray,
            N_cap: int, zero_pad: bool = True, x_perm_init: np.ndarray | None = None) -> dict:
    """Expert-grouped copy of the token rows plus both row maps."""
    x_bf16 = _c(x_bf16, np.uint16)
    topk_idx = _c(topk_idx, np.int64)
    expert_offsets = _c(expert_offsets, np.int32)
    T, H = x_bf16.shape
    K = topk_idx.shape[1]
    if x_perm_init is None:
        x_perm = np.zeros((N_cap, H), np.uint16)
    else:
        x_perm = np.array(x_perm_init, dtype=np.uint16, copy=True, order="C")
    r2f = np.empty(N_cap, np.int32)
    f2r = np.empty((T, K), np.int32)
    st = _load().oracle_permute(_p(x_bf16), _p(topk_idx), T, K, E, H, _p(expert_offsets),
                                int(bool(zero_pad)), N_cap, _p(x_perm), _p(r2f), _p(f2r))
    return dict(x_perm=x_perm, row_to_flat=r2f, flat_to_row=f2r, status=st)


def bruteforce_rows(topk_idx: np.ndarray, E: int, expert_offsets: np.ndarray) -> np.ndarray:
    topk_idx = _c(topk_idx, np.int64)
    expert_offsets = _c(expert_offsets, np.int32)
    T, K = topk_idx.shape
    rows = np.empty((T, K), np.int32)
    _load().oracle_bruteforce_rows(_p(topk_idx), T, K, E, _p(expert_offsets), _p(rows))
    return rows


# ------------------------------------------------------- stand-in expert ---

def expert_scale(rows_bf16: np.ndarray, expert_offsets: np.ndarray, tokens_per_expert: np.ndarray,
                 scales: np.ndarray, out_init: np.ndarray | None = None) -> np.ndarray:
    """y = bf16_rn(fp32(x) * s_e) over the real rows of each expert; pad rows 0."""
    rows_bf16 = _c(rows_bf16, np.uint16)
    expert_offsets = _c(expert_offsets, np.int32)
    tokens_per_expert = _c(tokens_per_expert, np.int32)
    scales = _c(scales, np.float32)
    E = scales.shape[0]
    H = rows_bf16.shape[1]
    out = np.zeros_like(rows_bf16) if out_init is None else np.array(out_init, np.uint16, copy=True)
    _load().oracle_expert_scale(_p(rows_bf16), _p(expert_offsets), _p(tokens_per_expert), E, H,
                                _p(scales), _p(out))
    return out


# --------------------------------------------------------------- combine ---

def combine(rows_bf16: np.ndarray, flat_to_row: np.ndarray, weights: np.ndarray | None,
            seq: bool = True) -> dict:
    """fused_weighted_restore: fp64 reference sum and (optionally) the FP32
    fmaf-chain value rounded to bf16.  weights=None means unit weights."""
    rows_bf16 = _c(rows_bf16, np.uint16)
    flat_to_row = _c(flat_to_row, np.int32)
    T, K = flat_to_row.shape
    N_cap, H = rows_bf16.shape
    w = None if weights is None else _c(np.asarray(weights, np.float32), np.float32)
    ref = np.empty((T, H), np.float64)
    out_seq = np.empty((T, H), np.uint16) if seq else None
    st = _load().oracle_combine(_p(rows_bf16), N_cap, _p(flat_to_row), _p(w), T, K, H, _p(ref),
                                _p(out_seq))
    return dict(ref=ref, seq=out_seq, status=st)


def check_coverage(row_to_flat: np.ndarray, flat_to_row: np.ndarray) -> int:
    row_to_flat = _c(row_to_flat, np.int32)
    flat_to_row = _c(flat_to_row, np.int32)
    return _load().oracle_check_coverage(_p(row_to_flat), _p(flat_to_row), row_to_flat.shape[0],
                                         flat_to_row.size)


def scatter_flat_index(row_flat: np.ndarray, T: int, K: int) -> dict:
    """flat_to_row [T,K] from the flat index each gathered row holds, with
    the coverage check of the folded restore."""
    row_flat = _c(row_flat, np.int32)
    f2r = np.empty((T, K), np.int32)
    st = _load().oracle_scatter_flat_index(_p(row_flat), row_flat.shape[0], T * K, _p(f2r))
    return dict(flat_to_row=f2r, status=st)


def combine_backward(grad_out_bf16: np.ndarray, rows_bf16: np.ndarray, row_to_flat: np.ndarray,
                     flat_to_row: np.ndarray, weights: np.ndarray, expert_offsets: np.ndarray,
                     zero_pad: bool = True, grad_rows_init: np.ndarray | None = None,
                     want_grad_w: bool = True) -> dict:
    """Row gradients bf16_rn(fp32(w*g)) and fp64 weight gradients <g_t, y_row>."""
    g = _c(grad_out_bf16, np.uint16)
    rows_bf16 = _c(rows_bf16, np.uint16)
    row_to_flat = _c(row_to_flat, np.int32)
    flat_to_row = _c(flat_to_row, np.int32)
    expert_offsets = _c(expert_offsets, np.int32)
    w = _c(np.asarray(weights, np.float32), np.float32)
    T, K = flat_to_row.shape
    N_cap, H = rows_bf16.shape
    E = expert_offsets.shape[0] - 1
    if grad_rows_init is None:
        grad_rows = np.zeros((N_cap, H), np.uint16)
    else:
        grad_rows = np.array(grad_rows_init, np.uint16, copy=True, order="C")
    grad_w = np.empty((T, K), np.float64) if want_grad_w else None
    st = _load().oracle_combine_backward(_p(g), _p(rows_bf16), N_cap, _p(row_to_flat),
                                         _p(flat_to_row), _p(w), T, K, H, _p(expert_offsets), E,
                                         int(bool(zero_pad)), _p(grad_rows), _p(grad_w))
    return dict(grad_rows=grad_rows, grad_w=grad_w, status=st)


# ----------------------------------------------- payload and fp32 variants ---

def permute_payload(x: np.ndarray, topk_idx: np.ndarray, E: int, expert_offsets: np.ndarray,
                    N_cap: int, aux: np.ndarray | None = None, zero_pad: bool = True,
                    x_perm_init: np.ndarray | None = None,
                    aux_perm_init: np.ndarray | None = None) -> dict:
    """Dispatch of opaque row payloads: x [T, ...] (any dtype, each token row
    row_bytes bytes) and optionally aux [T, ...] (e.g. FP8 scales)."""
    x = np.ascontiguousarray(x)
    topk_idx = _c(topk_idx, np.int64)
    expert_offsets = _c(expert_offsets, np.int32)
    T = x.shape[0]
    K = topk_idx.shape[1]
    row_bytes = x.nbytes // T if T else x.dtype.itemsize * int(np.prod(x.shape[1:]))
    shape = (N_cap,) + x.shape[1:]
    xp = (np.zeros(shape, x.dtype) if x_perm_init is None
          else np.array(x_perm_init, dtype=x.dtype, copy=True, order="C"))
    auxp, aux_bytes = None, 0
    if aux is not None:
        aux = np.ascontiguousarray(aux)
        aux_bytes = aux.nbytes // T if T else aux.dtype.itemsize * int(np.prod(aux.shape[1:]))
        ashape = (N_cap,) + aux.shape[1:]
        auxp = (np.zeros(ashape, aux.dtype) if aux_perm_init is None
                else np.array(aux_perm_init, dtype=aux.dtype, copy=True, order="C"))
    r2f = np.empty(N_cap, np.int32)
    f2r = np.empty((T, K), np.int32)
    st = _load().oracle_permute_payload(_p(x), row_bytes, _p(aux), aux_bytes, _p(topk_idx), T, K, E,
                                        _p(expert_offsets), int(bool(zero_pad)), N_cap, _p(xp),
                                        _p(auxp), _p(r2f), _p(f2r))
    return dict(x_perm=xp, aux_perm=auxp, row_to_flat=r2f, flat_to_row=f2r, status=st)


def combine_f32(rows: np.ndarray, flat_to_row: np.ndarray, weights: np.ndarray | None,
                seq: bool = True) -> dict:
    """fused_weighted_restore on fp32 rows: fp64 reference and the FP32
    fmaf-chain value (fp32 output)."""
    rows = _c(rows, np.float32)
    flat_to_row = _c(flat_to_row, np.int32)
    T, K = flat_to_row.shape
    N_cap, H = rows.shape
    w = None if weights is None else _c(np.asarray(weights, np.float32), np.float32)
    ref = np.empty((T, H), np.float64)
    out_seq = np.empty((T, H), np.float32) if seq else None
    st = _load().oracle_combine_f32(_p(rows), N_cap, _p(flat_to_row), _p(w), T, K, H, _p(ref),
                                    _p(out_seq))
    return dict(ref=ref, seq=out_seq, status=st)


def combine_backward_f32(grad_out: np.ndarray, rows: np.ndarray, row_to_flat: np.ndarray,
                         flat_to_row: np.ndarray, weights: np.ndarray, expert_offsets: np.ndarray,
                         zero_pad: bool = True, grad_rows_init: np.ndarray | None = None,
                         want_grad_w: bool = True) -> dict:
    """Row gradients fp32(w*g) and fp64 weight gradients <g_t, y_row> for
    fp32 rows."""
    g = _c(grad_out, np.float32)
    rows = _c(rows, np.float32)
    row_to_flat = _c(row_to_flat, np.int32)
    flat_to_row = _c(flat_to_row, np.int32)
    expert_offsets = _c(expert_offsets, np.int32)
    w = _c(np.asarray(weights, np.float32), np.float32)
    T, K = flat_to_row.shape
    N_cap, H = rows.shape
    E = expert_offsets.shape[0] - 1
    grad_rows = (np.zeros((N_cap, H), np.float32) if grad_rows_init is None
                 else np.array(grad_rows_init, np.float32, copy=True, order="C"))
    grad_w = np.empty((T, K), np.float64) if want_grad_w else None
    st = _load().oracle_combine_backward_f32(_p(g), _p(rows), N_cap, _p(row_to_flat),
                                             _p(flat_to_row), _p(w), T, K, H, _p(expert_offsets), E,
                                             int(bool(zero_pad)), _p(grad_rows), _p(grad_w))
    return dict(grad_rows=grad_rows, grad_w=grad_w, status=st)


def restore_activation_dtype(rows_bf16: np.ndarray, flat_to_row: np.ndarray, weights: np.ndarray,
                             grad_out_bf16: np.ndarray | None = None) -> dict:
    """The default (non-fused) folded restore: weights cast to bf16, every
    product and top-k addition rounded to bf16; optional score gradient
    through the bf16 weights.  An accuracy comparison only."""
    rows_bf16 = _c(rows_bf16, np.uint16)
    flat_to_row = _c(flat_to_row, np.int32)
    T, K = flat_to_row.shape
    N_cap, H = rows_bf16.shape
    w = _c(np.asarray(weights, np.float32), np.float32)
    g = None if grad_out_bf16 is None else _c(grad_out_bf16, np.uint16)
    out = np.empty((T, H), np.uint16)
    gw = np.empty((T, K), np.uint16) if g is not None else None
    st = _load().oracle_restore_activation_dtype(_p(rows_bf16), N_cap, _p(flat_to_row), _p(w), _p(g),
                                                 T, K, H, _p(out), _p(gw))
    return dict(out=out, grad_w=gw, status=st)

