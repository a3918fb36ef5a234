"""Split plan for expert parallelism across processes (one GPU per rank).

Source: DeepSpeed PR "Derive AutoEP rank splits from the per-expert count
exchange" (Redundancy, Fix, Tests).  Each rank knows how many of its own
assignments go to every (destination rank, local expert): its count matrix
[ep_size, E_local].  ONE all-to-all of that matrix gives every rank, as a
destination, the received counts [ep_size, E_local] (row s: what source rank
s sends to each of this rank's local experts); the row sums of the two
matrices are the rows this rank sends to / receives from each rank, and
received_counts.sum(dim=1) == output_splits holds exactly because one is
computed from the other.  The two split vectors come to the host in ONE
device-to-host copy (the payload all-to-all needs them as host integers).

On one GPU the library's layout computes the same quantities for all logical
ranks at once (counts [R, R, E_local], splits [R, R]); this module is the
exchange step a real multi-GPU deployment puts between the layout and the
payload all-to-all.  It is host plumbing over torch.distributed (NCCL on
GPUs, gloo on CPU); the per-expert counts of split_plan_from_expert_indices
come from the library's layout kernel.
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist

from . import api


@dataclasses.dataclass
class SplitPlan:
    """The plan of one rank.  (The page counts four fields without naming
    them; these are the four the exchange determines.)"""
    input_splits: list          # rows this rank sends to each destination rank (host ints)
    output_splits: list         # rows this rank receives from each source rank (host ints)
    received_counts: torch.Tensor           # [ep_size, E_local] int32, this rank as destination
    tokens_per_local_expert: torch.Tensor   # [E_local]: received_counts.sum(dim=0)


def count_matrix(tokens_per_expert: torch.Tensor, ep_size: int) -> torch.Tensor:
    """This rank's per-expert counts [E] viewed as [ep_size, E_local]: experts
    are contiguous blocks of E_local per destination rank."""
    E = tokens_per_expert.numel()
    if ep_size < 1 or E % ep_size:
        raise ValueError(f"{E} experts do not split into {ep_size} ranks")
    return tokens_per_expert.reshape(ep_size, E // ep_size)


def split_plan(counts: torch.Tensor, group=None) -> SplitPlan:
    """One all-to-all of the count matrix, one device-to-host copy."""
    ep_size = dist.get_world_size(group)
    if counts.dim() != 2 or counts.shape[0] != ep_size:
        raise ValueError(f"count matrix must be [ep_size={ep_size}, E_local], got "
                         f"{tuple(counts.shape)}")
    send = counts.to(torch.int32).contiguous()
    received = torch.empty_like(send)
    dist.all_to_all_single(received.view(-1), send.view(-1), group=group)
    both = torch.stack((send.sum(dim=1), received.sum(dim=1))).cpu()
    return SplitPlan(input_splits=both[0].tolist(), output_splits=both[1].tolist(),
                     received_counts=received, tokens_per_local_expert=received.sum(dim=0))


def split_plan_from_expert_indices(topk_idx: torch.Tensor, num_experts: int, group=None,
                                   status: torch.Tensor | None = None) -> SplitPlan:
    """The same plan straight from this rank's routing topk_idx [T_local, K]:
    the per-expert counts come from the library's layout kernel (this rank's
    tokens as one source block), then split_plan."""
    ep_size = dist.get_world_size(group)
    lay = api.dispatch_layout(topk_idx, num_experts, 1, 1, status=status)
    return split_plan(count_matrix(lay.tokens_per_expert, ep_size), group)
