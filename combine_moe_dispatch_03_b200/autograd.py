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
        lay = api.dispatch_layout(topk_idx, num_experts, num_ranks, align, status=status)
        x_perm, r2f, f2r = api.permute(x, topk_idx, lay, status=status)
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
