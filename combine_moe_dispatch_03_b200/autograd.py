"""Autograd wrapper over the dispatch -> stand-in experts -> combine chain.

Written the way the DeepEP issue "Does Deepep's Dispatch/Combine Support
Autograd Like PyTorch's all_to_all?" prescribes: a torch.autograd.Function
whose forward runs dispatch then combine, and whose backward runs the
combine's backward (a dispatch of the output gradient, here weighted, plus
the routing-weight gradient of fused_weighted_restore) and then the
dispatch's backward (a combine with unit weights).  Every step runs in the
library's kernels; this module only orders the calls.
"""
from __future__ import annotations

import torch

from . import api


class MoEDispatchCombine(torch.autograd.Function):
    """out = combine(stand_in_experts(dispatch(x)), weights).

    Inputs: x [T,H] bf16, topk_idx [T,K] int64, weights [T,K] fp32/bf16
    (router dtype), scales [E] fp32 (stand-in y = x*s_e), and the layout
    parameters.  Gradients flow to x and weights.
    """

    @staticmethod
    def forward(ctx, x, topk_idx, weights, scales, num_experts: int, num_ranks: int = 1,
                align: int = 1, validate: bool = False):
        status = api.new_status(x.device)
        lay, x_perm, r2f, f2r = api.dispatch(x, topk_idx, num_experts, num_ranks, align,
                                             status=status)
        y = api.expert_scale(x_perm, lay, scales, status=status)
        out = api.combine_weighted(y, f2r, weights, row_to_flat=r2f, validate=validate,
                                   status=status)
        ctx.save_for_backward(y, r2f, f2r, weights, scales, status)
        ctx.layout = lay
        ctx.mark_non_differentiable(status)
        return out, status

    @staticmethod
    def backward(ctx, grad_out, _grad_status):
        y, r2f, f2r, weights, scales, status = ctx.saved_tensors
        lay = ctx.layout
        grad_rows, grad_w = api.combine_backward(grad_out.contiguous(), y, r2f, f2r, weights, lay,
                                                 want_grad_weights=ctx.needs_input_grad[2],
                                                 status=status)
        grad_x = None
        if ctx.needs_input_grad[0]:
            grad_xp = api.expert_scale(grad_rows, lay, scales, status=status)
            grad_x = api.combine_weighted(grad_xp, f2r, None, status=status)
        return grad_x, None, grad_w, None, None, None, None, None


def moe_dispatch_combine(x, topk_idx, weights, scales, num_experts, num_ranks=1, align=1,
                         validate=False):
    """Functional form; returns (out, status).  Call api.check_status(status)
    when a host-side check is wanted (one synchronisation)."""
    return MoEDispatchCombine.apply(x, topk_idx, weights, scales, num_experts, num_ranks, align,
                                    validate)


# ------------------------------------------------ dispatch and combine apart ---
#
# The same two halves as separate autograd Functions, so that the caller's
# own experts (a grouped GEMM, an MLP over the expert-grouped buffer) sit
# between them.  This is the split the DeepEP issue recommends: dispatch's
# backward is a combine of the gradient with unit weights; combine's
# backward is a dispatch of the output gradient (weighted) plus the
# routing-weight gradient.


class DispatchHandle:
    """What dispatch leaves for combine and for both backwards (the part of
    DeepEP's ``handle``): the layout, both row maps and the status word."""

    def __init__(self, layout: api.Layout, row_to_flat: torch.Tensor, flat_to_row: torch.Tensor,
                 status: torch.Tensor):
        self.layout = layout
        self.row_to_flat = row_to_flat
        self.flat_to_row = flat_to_row
        self.status = status

    @property
    def num_rows(self) -> int:
        """Rows of the expert-grouped buffers (the worst-case capacity)."""
        return int(self.row_to_flat.shape[0])


class MoEDispatch(torch.autograd.Function):
    """x [T,H] -> x_perm [N_cap,H] in the handle's expert-grouped order."""

    @staticmethod
    def forward(ctx, x, topk_idx, handle: DispatchHandle):
        x_perm, _, _ = api.permute(x, topk_idx, handle.layout, capacity=handle.num_rows,
                                   status=handle.status,
                                   out=(torch.empty(handle.num_rows, x.shape[1], dtype=x.dtype,
                                                    device=x.device),
                                        handle.row_to_flat, handle.flat_to_row))
        ctx.handle = handle
        return x_perm

    @staticmethod
    def backward(ctx, grad_x_perm):
        h = ctx.handle
        grad_x = api.combine_weighted(grad_x_perm.contiguous(), h.flat_to_row, None,
                                      status=h.status)
        return grad_x, None, None


class MoECombine(torch.autograd.Function):
    """y [N_cap,H] (expert outputs in the handle's order), weights [T,K] ->
    out [T,H] = fused_weighted_restore."""

    @staticmethod
    def forward(ctx, y, weights, handle: DispatchHandle, validate: bool = False):
        out = api.combine_weighted(y, handle.flat_to_row, weights, row_to_flat=handle.row_to_flat,
                                   validate=validate, status=handle.status)
        ctx.save_for_backward(y, weights)
        ctx.handle = handle
        return out

    @staticmethod
    def backward(ctx, grad_out):
        y, weights = ctx.saved_tensors
        h = ctx.handle
        grad_y, grad_w = api.combine_backward(grad_out.contiguous(), y, h.row_to_flat,
                                              h.flat_to_row, weights, h.layout,
                                              want_grad_weights=ctx.needs_input_grad[1],
                                              status=h.status)
        return (grad_y if ctx.needs_input_grad[0] else None), grad_w, None, None


def dispatch(x, topk_idx, num_experts: int, num_ranks: int = 1, align: int = 1,
             status: torch.Tensor | None = None):
    """Layout + permute.  Returns (x_perm [N_cap,H], handle); N_cap is the
    worst case A + E*(align-1), so no host wait for the real row count.
    Expert e owns rows [off[e], off[e+1]) of x_perm, off =
    handle.layout.expert_offsets (its first tokens_per_expert[e] rows real,
    the rest zero padding).  Rows past the padded total off[E] hold
    unspecified values and are never read by combine or by either backward,
    so an expert should compute on the groups only, as a grouped GEMM over
    these offsets does."""
    st = status if status is not None else api.new_status(x.device)
    lay = api.dispatch_layout(topk_idx, num_experts, num_ranks, align, status=st)
    T, K = topk_idx.shape
    N = api.worst_case_rows(T, K, num_experts, align)
    handle = DispatchHandle(lay, torch.empty(N, dtype=torch.int32, device=x.device),
                            torch.empty(T, K, dtype=torch.int32, device=x.device), st)
    return MoEDispatch.apply(x, topk_idx, handle), handle


def combine(y, handle: DispatchHandle, weights, validate: bool = False):
    """fused_weighted_restore of the expert outputs; differentiable in y and
    weights.  Call api.check_status(handle.status) for a host-side check."""
    return MoECombine.apply(y, weights, handle, validate)
