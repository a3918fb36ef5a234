"""Python entry points over the C ABI -- argument marshalling only.

Every function takes CUDA tensors, allocates its outputs with torch (device
memory from the caching allocator, no host synchronisation), and enqueues the
library's kernels on the current torch stream.  Device-side errors accumulate
in an int32 ``status`` tensor; ``check_status`` reads it (one sync) and raises
a RuntimeError naming the bits, the way the coverage check of
fused_weighted_restore raises (DeepSpeed PR "AutoEP: support
combine_impl=fused_weighted_sum with AutoEP+AutoTP folding", Change).

The names follow the C ABI: dispatch_layout / permute / expert_scale /
combine_weighted / combine_backward.  A ``Layout`` plus the two row maps play
the part of DeepEP's dispatch ``handle`` (DeepEP issue "Does Deepep's
Dispatch/Combine Support Autograd Like PyTorch's all_to_all?").
"""
from __future__ import annotations

import dataclasses
import math

import torch

from . import _lib
from ._lib import DTYPE_BF16, DTYPE_F32, check_rc, lib


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _stream(device: torch.device):
    return torch.cuda.current_stream(device).cuda_stream


def _require(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int | None = None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def _check_out(t: torch.Tensor, name: str, shape: tuple, dtype: torch.dtype, device):
    """A caller-provided output (or a tensor whose size another fixes): the
    kernels write/read exactly `shape`, so anything else is refused here,
    before any launch."""
    _require(t, name, dtype)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _check_layout(layout: "Layout", T: int, K: int, device):
    if layout.T != T or layout.K != K:
        raise ValueError(f"layout was built for T={layout.T}, K={layout.K}; got T={T}, K={K}")
    if layout.expert_offsets.device != device:
        raise ValueError(f"layout is on {layout.expert_offsets.device}, expected {device}")


def _weight_dtype(w: torch.Tensor) -> int:
    if w.dtype == torch.float32:
        return DTYPE_F32
    if w.dtype == torch.bfloat16:
        return DTYPE_BF16
    raise TypeError(f"weights must be float32 or bfloat16 (router dtype), got {w.dtype}")


def new_status(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def check_status(status: torch.Tensor) -> None:
    """Synchronise once on ``status`` and raise if any kernel flagged bad data."""
    bits = int(status.item())
    if bits:
        raise RuntimeError("MoE dispatch/combine device check failed: "
                           + "; ".join(_lib.decode_status(bits)) + f" (status bits {bits:#x})")


def worst_case_rows(T: int, K: int, E: int, align: int) -> int:
    n = lib().moe_worst_case_rows(T, K, E, align)
    if n < 0:
        raise ValueError("invalid sizes")
    return int(n)


def workspace_bytes(T: int, K: int, E: int, R: int) -> int:
    n = lib().moe_layout_workspace_bytes(T, K, E, R)
    if n == 0:
        raise ValueError("invalid sizes for the layout workspace")
    return int(n)


@dataclasses.dataclass
class Layout:
    """Outputs of moe_dispatch_layout (all device tensors)."""
    tokens_per_expert: torch.Tensor   # [E] int32
    counts: torch.Tensor              # [R, R, E/R] int32
    splits: torch.Tensor              # [R, R] int32
    tokens_per_rank: torch.Tensor     # [R, R] int32
    is_token_in_rank: torch.Tensor    # [T, R] uint8
    expert_offsets: torch.Tensor      # [E+1] int32
    workspace: torch.Tensor           # opaque, uint8
    T: int
    K: int
    E: int
    R: int
    align: int


def alloc_layout(T: int, K: int, E: int, R: int, align: int, device) -> Layout:
    i32 = dict(dtype=torch.int32, device=device)
    return Layout(
        tokens_per_expert=torch.empty(E, **i32),
        counts=torch.empty(R, R, E // R, **i32),
        splits=torch.empty(R, R, **i32),
        tokens_per_rank=torch.empty(R, R, **i32),
        is_token_in_rank=torch.empty(T, R, dtype=torch.uint8, device=device),
        expert_offsets=torch.empty(E + 1, **i32),
        workspace=torch.empty(workspace_bytes(T, K, E, R), dtype=torch.uint8, device=device),
        T=T, K=K, E=E, R=R, align=align)


def dispatch_layout(topk_idx: torch.Tensor, num_experts: int, num_ranks: int = 1,
                    align: int = 1, status: torch.Tensor | None = None,
                    out: Layout | None = None) -> Layout:
    _require(topk_idx, "topk_idx", torch.int64, 2)
    T, K = topk_idx.shape
    dev = topk_idx.device
    if out is not None and (out.T, out.K, out.E, out.R) != (T, K, num_experts, num_ranks):
        raise ValueError(f"out layout was allocated for (T, K, E, R) = {(out.T, out.K, out.E, out.R)}, "
                         f"got {(T, K, num_experts, num_ranks)}")
    if out is not None:
        out.align = align
    lay = out if out is not None else alloc_layout(T, K, num_experts, num_ranks, align, dev)
    st = status if status is not None else new_status(dev)
    rc = lib().moe_dispatch_layout(
        _ptr(topk_idx), T, K, num_experts, num_ranks, align, _ptr(lay.tokens_per_expert),
        _ptr(lay.counts), _ptr(lay.splits), _ptr(lay.tokens_per_rank), _ptr(lay.is_token_in_rank),
        _ptr(lay.expert_offsets), _ptr(lay.workspace), _ptr(st), _stream(dev))
    check_rc(rc, "moe_dispatch_layout")
    return lay


def permute(x: torch.Tensor, topk_idx: torch.Tensor, layout: Layout, capacity: int | None = None,
            zero_pad: bool = True, status: torch.Tensor | None = None,
            out: tuple | None = None):
    """Returns (x_perm [N_cap,H] bf16, row_to_flat [N_cap] int32, flat_to_row [T,K] int32)."""
    _require(x, "x", torch.bfloat16, 2)
    _require(topk_idx, "topk_idx", torch.int64, 2)
    T, H = x.shape
    K = topk_idx.shape[1]
    dev = x.device
    _check_out(topk_idx, "topk_idx", (T, K), torch.int64, dev)
    _check_layout(layout, T, K, dev)
    N_cap = capacity if capacity is not None else worst_case_rows(T, K, layout.E, layout.align)
    if out is None:
        x_perm = torch.empty(N_cap, H, dtype=torch.bfloat16, device=dev)
        r2f = torch.empty(N_cap, dtype=torch.int32, device=dev)
        f2r = torch.empty(T, K, dtype=torch.int32, device=dev)
    else:
        x_perm, r2f, f2r = out
        _check_out(x_perm, "x_perm", (N_cap, H), torch.bfloat16, dev)
        _check_out(r2f, "row_to_flat", (N_cap,), torch.int32, dev)
        _check_out(f2r, "flat_to_row", (T, K), torch.int32, dev)
    st = status if status is not None else new_status(dev)
    rc = lib().moe_permute(_ptr(x), _ptr(topk_idx), T, K, layout.E, H, _ptr(layout.expert_offsets),
                           _ptr(layout.workspace), int(bool(zero_pad)), N_cap, _ptr(x_perm),
                           _ptr(r2f), _ptr(f2r), _ptr(st), _stream(dev))
    check_rc(rc, "moe_permute")
    return x_perm, r2f, f2r


def dispatch(x: torch.Tensor, topk_idx: torch.Tensor, num_experts: int, num_ranks: int = 1,
             align: int = 1, capacity: int | None = None, zero_pad: bool = True,
             status: torch.Tensor | None = None, layout_out: Layout | None = None,
             out: tuple | None = None):
    """dispatch_layout and permute in one call (moe_dispatch).  Returns
    (layout, x_perm, row_to_flat, flat_to_row)."""
    _require(x, "x", torch.bfloat16, 2)
    _require(topk_idx, "topk_idx", torch.int64, 2)
    T, H = x.shape
    K = topk_idx.shape[1]
    dev = x.device
    _check_out(topk_idx, "topk_idx", (T, K), torch.int64, dev)
    E, R = num_experts, num_ranks
    if layout_out is not None and (layout_out.T, layout_out.K, layout_out.E, layout_out.R) != (T, K, E, R):
        raise ValueError(f"layout_out was allocated for (T, K, E, R) = "
                         f"{(layout_out.T, layout_out.K, layout_out.E, layout_out.R)}, got {(T, K, E, R)}")
    lay = layout_out if layout_out is not None else alloc_layout(T, K, E, R, align, dev)
    lay.align = align
    _check_layout(lay, T, K, dev)
    N_cap = capacity if capacity is not None else worst_case_rows(T, K, E, align)
    if out is None:
        x_perm = torch.empty(N_cap, H, dtype=torch.bfloat16, device=dev)
        r2f = torch.empty(N_cap, dtype=torch.int32, device=dev)
        f2r = torch.empty(T, K, dtype=torch.int32, device=dev)
    else:
        x_perm, r2f, f2r = out
        _check_out(x_perm, "x_perm", (N_cap, H), torch.bfloat16, dev)
        _check_out(r2f, "row_to_flat", (N_cap,), torch.int32, dev)
        _check_out(f2r, "flat_to_row", (T, K), torch.int32, dev)
    st = status if status is not None else new_status(dev)
    rc = lib().moe_dispatch(
        _ptr(x), _ptr(topk_idx), T, K, E, R, H, align, _ptr(lay.tokens_per_expert),
        _ptr(lay.counts), _ptr(lay.splits), _ptr(lay.tokens_per_rank), _ptr(lay.is_token_in_rank),
        _ptr(lay.expert_offsets), _ptr(lay.workspace), int(bool(zero_pad)), N_cap, _ptr(x_perm),
        _ptr(r2f), _ptr(f2r), _ptr(st), _stream(dev))
    check_rc(rc, "moe_dispatch")
    return lay, x_perm, r2f, f2r


def expert_scale(rows: torch.Tensor, layout: Layout, scales: torch.Tensor,
                 status: torch.Tensor | None = None, out: torch.Tensor | None = None):
    """Stand-in expert: y = bf16_rn(rows * s_e) on real rows, 0 on pad rows."""
    _require(rows, "rows", torch.bfloat16, 2)
    _require(scales, "scales", torch.float32, 1)
    N_cap, H = rows.shape
    _check_out(scales, "scales", (layout.E,), torch.float32, rows.device)
    if layout.expert_offsets.device != rows.device:
        raise ValueError("layout and rows are on different devices")
    y = out if out is not None else torch.empty_like(rows)
    _check_out(y, "out", (N_cap, H), torch.bfloat16, rows.device)
    st = status if status is not None else new_status(rows.device)
    rc = lib().moe_expert_scale(_ptr(rows), N_cap, _ptr(layout.expert_offsets),
                                _ptr(layout.tokens_per_expert), layout.E, H, _ptr(scales), _ptr(y),
                                _ptr(st), _stream(rows.device))
    check_rc(rc, "moe_expert_scale")
    return y


def combine_weighted(rows: torch.Tensor, flat_to_row: torch.Tensor,
                     weights: torch.Tensor | None = None, row_to_flat: torch.Tensor | None = None,
                     validate: bool = False, status: torch.Tensor | None = None,
                     out: torch.Tensor | None = None):
    """fused_weighted_restore; weights=None is the unit-weight combine
    (the backward of dispatch).  bf16 rows give a bf16 output (FP32
    accumulation, one rounding); fp32 rows an fp32 output."""
    if isinstance(rows, torch.Tensor) and rows.dtype == torch.float32:
        return _combine_weighted_f32(rows, flat_to_row, weights, row_to_flat, validate, status, out)
    _require(rows, "rows", torch.bfloat16, 2)
    _require(flat_to_row, "flat_to_row", torch.int32, 2)
    N_cap, H = rows.shape
    T, K = flat_to_row.shape
    wd = DTYPE_F32
    if weights is not None:
        wd = _weight_dtype(weights)
        _require(weights, "weights", weights.dtype, 2)
        if tuple(weights.shape) != (T, K):
            raise ValueError("weights must be [T, K]")
    if validate:
        if row_to_flat is None:
            raise ValueError("validate=True needs row_to_flat")
        _check_out(row_to_flat, "row_to_flat", (N_cap,), torch.int32, rows.device)
    if flat_to_row.device != rows.device or (weights is not None and weights.device != rows.device):
        raise ValueError("rows, flat_to_row and weights must be on one device")
    o = out if out is not None else torch.empty(T, H, dtype=torch.bfloat16, device=rows.device)
    _check_out(o, "out", (T, H), torch.bfloat16, rows.device)
    st = status if status is not None else new_status(rows.device)
    rc = lib().moe_combine_weighted(_ptr(rows), N_cap, _ptr(row_to_flat), _ptr(flat_to_row),
                                    _ptr(weights), wd, T, K, H, int(bool(validate)), _ptr(o),
                                    _ptr(st), _stream(rows.device))
    check_rc(rc, "moe_combine_weighted")
    return o


def combine_backward(grad_out: torch.Tensor, rows: torch.Tensor, row_to_flat: torch.Tensor,
                     flat_to_row: torch.Tensor, weights: torch.Tensor, layout: Layout,
                     zero_pad: bool = True, want_grad_weights: bool = True,
                     status: torch.Tensor | None = None, out: tuple | None = None):
    """Returns (grad_rows [N_cap,H] in the rows' dtype (bf16 or fp32),
    grad_weights [T,K] router dtype or None)."""
    if isinstance(rows, torch.Tensor) and rows.dtype == torch.float32:
        return _combine_backward_f32(grad_out, rows, row_to_flat, flat_to_row, weights, layout,
                                     zero_pad, want_grad_weights, status, out)
    _require(grad_out, "grad_out", torch.bfloat16, 2)
    _require(rows, "rows", torch.bfloat16, 2)
    _require(flat_to_row, "flat_to_row", torch.int32, 2)
    _require(row_to_flat, "row_to_flat", torch.int32, 1)
    wd = _weight_dtype(weights)
    _require(weights, "weights", weights.dtype, 2)
    N_cap, H = rows.shape
    T, K = flat_to_row.shape
    dev = rows.device
    _check_out(grad_out, "grad_out", (T, H), torch.bfloat16, dev)
    _check_out(row_to_flat, "row_to_flat", (N_cap,), torch.int32, dev)
    _check_out(weights, "weights", (T, K), weights.dtype, dev)
    _check_out(flat_to_row, "flat_to_row", (T, K), torch.int32, dev)
    if layout.expert_offsets.device != dev:
        raise ValueError("layout and rows are on different devices")
    if out is None:
        grad_rows = torch.empty_like(rows)
        grad_w = torch.empty(T, K, dtype=weights.dtype, device=rows.device) if want_grad_weights else None
    else:
        grad_rows, grad_w = out
        _check_out(grad_rows, "grad_rows", (N_cap, H), torch.bfloat16, dev)
        if grad_w is not None:
            _check_out(grad_w, "grad_weights", (T, K), weights.dtype, dev)
    st = status if status is not None else new_status(rows.device)
    rc = lib().moe_combine_backward(_ptr(grad_out), _ptr(rows), N_cap, _ptr(row_to_flat),
                                    _ptr(flat_to_row), _ptr(weights), wd, T, K, H,
                                    _ptr(layout.expert_offsets), layout.E, int(bool(zero_pad)),
                                    _ptr(grad_rows), _ptr(grad_w), _ptr(st), _stream(rows.device))
    check_rc(rc, "moe_combine_backward")
    return grad_rows, grad_w


def scatter_flat_index(row_flat: torch.Tensor, T: int, K: int,
                       status: torch.Tensor | None = None, out: torch.Tensor | None = None):
    """flat_to_row [T,K] from the flat index each gathered row holds (-1: none),
    with the folded restore's coverage check (MOE_ST_COVERAGE)."""
    _require(row_flat, "row_flat", torch.int32, 1)
    f2r = out if out is not None else torch.empty(T, K, dtype=torch.int32, device=row_flat.device)
    _check_out(f2r, "out", (T, K), torch.int32, row_flat.device)
    st = status if status is not None else new_status(row_flat.device)
    rc = lib().moe_scatter_flat_index(_ptr(row_flat), row_flat.shape[0], T, K, _ptr(f2r),
                                      _ptr(st), _stream(row_flat.device))
    check_rc(rc, "moe_scatter_flat_index")
    return f2r


def segment_labels(counts: torch.Tensor, modulo: int, rows: int,
                   status: torch.Tensor | None = None, out: torch.Tensor | None = None):
    """labels [rows] int64: row i of n consecutive segments (segment j holding
    counts[j] rows) gets j % modulo; rows past sum(counts) get -1."""
    _require(counts, "counts", torch.int32, 1)
    dev = counts.device
    lab = out if out is not None else torch.empty(rows, dtype=torch.int64, device=dev)
    _check_out(lab, "out", (rows,), torch.int64, dev)
    st = status if status is not None else new_status(dev)
    rc = lib().moe_segment_labels(_ptr(counts), counts.shape[0], modulo, rows, _ptr(lab), _ptr(st),
                                  _stream(dev))
    check_rc(rc, "moe_segment_labels")
    return lab


def rank_bases(all_counts: torch.Tensor, rank: int, align: int = 1,
               status: torch.Tensor | None = None, out: tuple | None = None):
    """moe_rank_bases: from the per-expert counts of every source rank
    (all_counts [R, E] int32, on the device) the row bases of the direct
    dispatch for `rank`.  Returns (dest_base [E], own_offsets [E/R + 1],
    own_counts [E/R], max_rows [1]) int32 device tensors."""
    _require(all_counts, "all_counts", torch.int32, 2)
    R, E = all_counts.shape
    if E % R:
        raise ValueError(f"{E} experts do not split into {R} ranks")
    dev = all_counts.device
    i32 = dict(dtype=torch.int32, device=dev)
    if out is None:
        out = (torch.empty(E, **i32), torch.empty(E // R + 1, **i32), torch.empty(E // R, **i32),
               torch.empty(1, **i32))
    dest_base, own_off, own_cnt, max_rows = out
    _check_out(dest_base, "dest_base", (E,), torch.int32, dev)
    _check_out(own_off, "own_offsets", (E // R + 1,), torch.int32, dev)
    _check_out(own_cnt, "own_counts", (E // R,), torch.int32, dev)
    _check_out(max_rows, "max_rows", (1,), torch.int32, dev)
    st = status if status is not None else new_status(dev)
    rc = lib().moe_rank_bases(_ptr(all_counts), R, E, rank, align, _ptr(dest_base), _ptr(own_off),
                              _ptr(own_cnt), _ptr(max_rows), _ptr(st), _stream(dev))
    check_rc(rc, "moe_rank_bases")
    return dest_base, own_off, own_cnt, max_rows


def permute_to_ranks(x: torch.Tensor, topk_idx: torch.Tensor, layout: Layout,
                     dest_base: torch.Tensor, dest_table: torch.Tensor, dest_cap: int, rank: int,
                     own_offsets: torch.Tensor, own_counts: torch.Tensor, zero_pad: bool = True,
                     claims_table: torch.Tensor | None = None,
                     status: torch.Tensor | None = None, out: torch.Tensor | None = None):
    """moe_permute_to_ranks: rows straight into the buffers listed in
    dest_table (int64 device tensor [R] of buffer addresses).  With
    claims_table (int64 device tensor [R] of int32 [dest_cap] array
    addresses) every stored row also records which (rank, token, slot) it
    holds, for the restore's coverage check.  Returns flat_to_row [T,K] (row
    in the buffer of each slot's expert rank)."""
    _require(x, "x", torch.bfloat16, 2)
    _require(topk_idx, "topk_idx", torch.int64, 2)
    T, H = x.shape
    K = topk_idx.shape[1]
    dev = x.device
    _check_out(topk_idx, "topk_idx", (T, K), torch.int64, dev)
    _check_layout(layout, T, K, dev)
    if layout.R != 1:
        raise ValueError("the layout must be of this rank's own tokens (num_ranks=1)")
    _require(dest_table, "dest_table", torch.int64, 1)
    R = dest_table.shape[0]
    E = layout.E
    if E % R:
        raise ValueError(f"{E} experts do not split into {R} ranks")
    _check_out(dest_base, "dest_base", (E,), torch.int32, dev)
    _check_out(own_offsets, "own_offsets", (E // R + 1,), torch.int32, dev)
    _check_out(own_counts, "own_counts", (E // R,), torch.int32, dev)
    if claims_table is not None:
        _check_out(claims_table, "claims_table", (R,), torch.int64, dev)
    f2r = out if out is not None else torch.empty(T, K, dtype=torch.int32, device=dev)
    _check_out(f2r, "flat_to_row", (T, K), torch.int32, dev)
    st = status if status is not None else new_status(dev)
    rc = lib().moe_permute_to_ranks(_ptr(x), _ptr(topk_idx), T, K, E, R, H, _ptr(dest_base),
                                    _ptr(layout.workspace), _ptr(dest_table), _ptr(claims_table),
                                    dest_cap, rank, _ptr(own_offsets), _ptr(own_counts),
                                    int(bool(zero_pad)), _ptr(f2r), _ptr(st), _stream(dev))
    check_rc(rc, "moe_permute_to_ranks")
    return f2r


def combine_from_ranks(rows_table: torch.Tensor, N_cap: int, H: int, flat_to_row: torch.Tensor,
                       topk_idx: torch.Tensor, num_experts: int, weights: torch.Tensor,
                       claims_table: torch.Tensor | None = None, rank: int = 0,
                       status: torch.Tensor | None = None, out: torch.Tensor | None = None):
    """moe_combine_from_ranks: fused_weighted_restore reading each slot's row
    from the buffer of its expert's rank (rows_table: int64 device tensor [R]
    of bf16 [N_cap, H] buffer addresses).  With claims_table (the one the
    dispatch filled) and this rank's index, every slot's row is checked to be
    claimed by this (rank, token, slot): MOE_ST_COVERAGE otherwise."""
    _require(rows_table, "rows_table", torch.int64, 1)
    _require(flat_to_row, "flat_to_row", torch.int32, 2)
    T, K = flat_to_row.shape
    dev = flat_to_row.device
    _check_out(topk_idx, "topk_idx", (T, K), torch.int64, dev)
    wd = _weight_dtype(weights)
    _check_out(weights, "weights", (T, K), weights.dtype, dev)
    o = out if out is not None else torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    _check_out(o, "out", (T, H), torch.bfloat16, dev)
    st = status if status is not None else new_status(dev)
    if claims_table is not None:
        _check_out(claims_table, "claims_table", (rows_table.shape[0],), torch.int64, dev)
    rc = lib().moe_combine_from_ranks(_ptr(rows_table), _ptr(claims_table), rows_table.shape[0],
                                      rank, N_cap, _ptr(flat_to_row), _ptr(topk_idx), num_experts,
                                      _ptr(weights), wd, T, K, H, _ptr(o), _ptr(st), _stream(dev))
    check_rc(rc, "moe_combine_from_ranks")
    return o


def _combine_weighted_f32(rows, flat_to_row, weights, row_to_flat, validate, status, out):
    _require(rows, "rows", torch.float32, 2)
    _require(flat_to_row, "flat_to_row", torch.int32, 2)
    N_cap, H = rows.shape
    T, K = flat_to_row.shape
    wd = DTYPE_F32
    if weights is not None:
        wd = _weight_dtype(weights)
        _require(weights, "weights", weights.dtype, 2)
        if tuple(weights.shape) != (T, K):
            raise ValueError("weights must be [T, K]")
    if validate:
        if row_to_flat is None:
            raise ValueError("validate=True needs row_to_flat")
        _check_out(row_to_flat, "row_to_flat", (N_cap,), torch.int32, rows.device)
    if flat_to_row.device != rows.device or (weights is not None and weights.device != rows.device):
        raise ValueError("rows, flat_to_row and weights must be on one device")
    o = out if out is not None else torch.empty(T, H, dtype=torch.float32, device=rows.device)
    _check_out(o, "out", (T, H), torch.float32, rows.device)
    st = status if status is not None else new_status(rows.device)
    rc = lib().moe_combine_weighted_f32(_ptr(rows), N_cap, _ptr(row_to_flat), _ptr(flat_to_row),
                                        _ptr(weights), wd, T, K, H, int(bool(validate)), _ptr(o),
                                        _ptr(st), _stream(rows.device))
    check_rc(rc, "moe_combine_weighted_f32")
    return o


def _combine_backward_f32(grad_out, rows, row_to_flat, flat_to_row, weights, layout, zero_pad,
                          want_grad_weights, status, out):
    _require(grad_out, "grad_out", torch.float32, 2)
    _require(rows, "rows", torch.float32, 2)
    _require(flat_to_row, "flat_to_row", torch.int32, 2)
    _require(row_to_flat, "row_to_flat", torch.int32, 1)
    wd = _weight_dtype(weights)
    _require(weights, "weights", weights.dtype, 2)
    N_cap, H = rows.shape
    T, K = flat_to_row.shape
    dev = rows.device
    _check_out(grad_out, "grad_out", (T, H), torch.float32, dev)
    _check_out(row_to_flat, "row_to_flat", (N_cap,), torch.int32, dev)
    _check_out(weights, "weights", (T, K), weights.dtype, dev)
    if layout.expert_offsets.device != dev:
        raise ValueError("layout and rows are on different devices")
    if out is None:
        grad_rows = torch.empty_like(rows)
        grad_w = torch.empty(T, K, dtype=weights.dtype, device=rows.device) if want_grad_weights else None
    else:
        grad_rows, grad_w = out
        _check_out(grad_rows, "grad_rows", (N_cap, H), torch.float32, dev)
        if grad_w is not None:
            _check_out(grad_w, "grad_weights", (T, K), weights.dtype, dev)
    st = status if status is not None else new_status(rows.device)
    rc = lib().moe_combine_backward_f32(_ptr(grad_out), _ptr(rows), N_cap, _ptr(row_to_flat),
                                        _ptr(flat_to_row), _ptr(weights), wd, T, K, H,
                                        _ptr(layout.expert_offsets), layout.E, int(bool(zero_pad)),
                                        _ptr(grad_rows), _ptr(grad_w), _ptr(st), _stream(rows.device))
    check_rc(rc, "moe_combine_backward_f32")
    return grad_rows, grad_w


def permute_payload(x: torch.Tensor, topk_idx: torch.Tensor, layout: Layout,
                    aux: torch.Tensor | None = None, capacity: int | None = None,
                    zero_pad: bool = True, status: torch.Tensor | None = None,
                    out: tuple | None = None):
    """Dispatch of an opaque row payload x [T, ...] (any dtype; e.g. the e4m3
    data of an FP8 tuple, or fp32 rows) and an optional per-token aux payload
    [T, ...] (e.g. the FP8 scales).  Returns (x_perm, aux_perm or None,
    row_to_flat, flat_to_row)."""
    if not isinstance(x, torch.Tensor) or not x.is_cuda or not x.is_contiguous() or x.dim() < 1:
        raise ValueError("x must be a contiguous CUDA tensor [T, ...]")
    _require(topk_idx, "topk_idx", torch.int64, 2)
    T = x.shape[0]
    K = topk_idx.shape[1]
    dev = x.device
    row_bytes = x.element_size() * math.prod(x.shape[1:])
    aux_bytes = 0
    if aux is not None:
        if not aux.is_cuda or not aux.is_contiguous() or aux.shape[0] != T:
            raise ValueError("aux must be a contiguous CUDA tensor [T, ...]")
        aux_bytes = aux.element_size() * math.prod(aux.shape[1:])
    _check_out(topk_idx, "topk_idx", (T, K), torch.int64, dev)
    _check_layout(layout, T, K, dev)
    N_cap = capacity if capacity is not None else worst_case_rows(T, K, layout.E, layout.align)
    if out is None:
        x_perm = torch.empty((N_cap,) + tuple(x.shape[1:]), dtype=x.dtype, device=dev)
        aux_perm = (torch.empty((N_cap,) + tuple(aux.shape[1:]), dtype=aux.dtype, device=dev)
                    if aux is not None else None)
        r2f = torch.empty(N_cap, dtype=torch.int32, device=dev)
        f2r = torch.empty(T, K, dtype=torch.int32, device=dev)
    else:
        x_perm, aux_perm, r2f, f2r = out
        _check_out(x_perm, "x_perm", (N_cap,) + tuple(x.shape[1:]), x.dtype, dev)
        if aux is not None:
            _check_out(aux_perm, "aux_perm", (N_cap,) + tuple(aux.shape[1:]), aux.dtype, dev)
        _check_out(r2f, "row_to_flat", (N_cap,), torch.int32, dev)
        _check_out(f2r, "flat_to_row", (T, K), torch.int32, dev)
    if aux is not None and aux.device != dev:
        raise ValueError("aux and x must be on one device")
    st = status if status is not None else new_status(dev)
    rc = lib().moe_permute_payload(_ptr(x), row_bytes, _ptr(aux), aux_bytes, _ptr(topk_idx), T, K,
                                   layout.E, _ptr(layout.expert_offsets), _ptr(layout.workspace),
                                   int(bool(zero_pad)), N_cap, _ptr(x_perm), _ptr(aux_perm),
                                   _ptr(r2f), _ptr(f2r), _ptr(st), _stream(dev))
    check_rc(rc, "moe_permute_payload")
    return x_perm, aux_perm, r2f, f2r
