"""Expert parallelism across processes (one GPU per rank): the split plan,
then dispatch and combine around the row exchange.

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
ranks at once (counts [R, R, E_local], splits [R, R]); this module is what a
multi-GPU deployment puts around the exchanges: the split plan, then the
rows (see the section "the payload across ranks" below).  Every step on the
rows runs in the library's kernels; the exchanges are torch.distributed
all-to-alls (NCCL on GPUs; the split plan also runs over gloo on CPU).
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


def plan_from_counts(counts: torch.Tensor, received: torch.Tensor) -> SplitPlan:
    """The plan from this rank's count matrix and the received counts (what
    the exchange delivers): row sums of both, one device-to-host copy."""
    both = torch.stack((counts.sum(dim=1), received.sum(dim=1))).cpu()
    return SplitPlan(input_splits=both[0].tolist(), output_splits=both[1].tolist(),
                     received_counts=received, tokens_per_local_expert=received.sum(dim=0))


def split_plan(counts: torch.Tensor, group=None) -> SplitPlan:
    """One all-to-all of the count matrix, one device-to-host copy."""
    ep_size = dist.get_world_size(group)
    if counts.dim() != 2 or counts.shape[0] != ep_size:
        raise ValueError(f"count matrix must be [ep_size={ep_size}, E_local], got "
                         f"{tuple(counts.shape)}")
    send = counts.to(torch.int32).contiguous()
    received = torch.empty_like(send)
    dist.all_to_all_single(received.view(-1), send.view(-1), group=group)
    return plan_from_counts(send, received)


def split_plan_from_expert_indices(topk_idx: torch.Tensor, num_experts: int, group=None,
                                   status: torch.Tensor | None = None) -> SplitPlan:
    """The same plan straight from this rank's routing topk_idx [T_local, K]:
    the per-expert counts come from the library's layout kernel (this rank's
    tokens as one source block), then split_plan."""
    ep_size = dist.get_world_size(group)
    lay = api.dispatch_layout(topk_idx, num_experts, 1, 1, status=status)
    return split_plan(count_matrix(lay.tokens_per_expert, ep_size), group)


# ---------------------------------------------- the payload across ranks ---
#
# Dispatch across ranks, as steps around the two exchanges:
#   send side:    layout of this rank's tokens (one source block, no padding)
#                 and permute: rows in (expert, token, slot) order, which is
#                 (destination rank, local expert, token, slot) because a
#                 rank's experts are contiguous -- so the permuted buffer IS
#                 the send buffer, input_splits[r] rows for rank r in turn;
#   exchange:     the split plan, then the rows (all-to-all-v);
#   receive side: rows arrive source by source, each source's rows in
#                 local-expert order; labelled with their local expert
#                 (moe_segment_labels over received_counts) they are regrouped
#                 by expert with a top_k = 1 layout + permute (stable: source
#                 rank, then token -- the order the single-GPU layout gives
#                 the same expert), padded to the grouped-GEMM alignment.
# Combine runs the same steps backwards: a unit-weight top_k = 1 combine
# ungroups the expert outputs into received order (an exact copy), the
# reverse exchange returns them to their source ranks in send order, and
# fused_weighted_restore over the send side's maps gives the output.


@dataclasses.dataclass
class EPHandle:
    """What dispatch across ranks leaves for combine."""
    send_layout: api.Layout
    send_row_to_flat: torch.Tensor      # [A]: send row -> (token, slot) of this rank
    send_flat_to_row: torch.Tensor      # [T_local, K]
    plan: SplitPlan
    recv_layout: api.Layout             # received rows by local expert (top_k = 1)
    recv_row_to_flat: torch.Tensor      # [N_grouped]: grouped row -> received row
    recv_flat_to_row: torch.Tensor      # [N_recv, 1]
    status: torch.Tensor


def dispatch_send(x: torch.Tensor, topk_idx: torch.Tensor, num_experts: int, ep_size: int,
                  status: torch.Tensor):
    """Send side: (send rows [A, H] in destination-rank order, layout,
    row_to_flat, flat_to_row, count matrix [ep_size, E_local])."""
    T, K = topk_idx.shape
    lay = api.dispatch_layout(topk_idx, num_experts, 1, 1, status=status)
    send, r2f, f2r = api.permute(x, topk_idx, lay, capacity=T * K, status=status)
    return send, lay, r2f, f2r, count_matrix(lay.tokens_per_expert, ep_size)


def dispatch_recv(recv_rows: torch.Tensor, plan: SplitPlan, align: int, status: torch.Tensor):
    """Receive side: (expert-grouped rows [N_recv + E_local*(align-1), H],
    layout, row_to_flat, flat_to_row) from the rows as they arrived."""
    n_recv = recv_rows.shape[0]
    E_local = plan.received_counts.shape[1]
    labels = api.segment_labels(plan.received_counts.reshape(-1), E_local, n_recv, status=status)
    rtopk = labels.view(n_recv, 1)
    rlay = api.dispatch_layout(rtopk, E_local, 1, align, status=status)
    grouped, rr2f, rf2r = api.permute(recv_rows, rtopk, rlay, status=status)
    return grouped, rlay, rr2f, rf2r


def combine_send(y_grouped: torch.Tensor, handle: EPHandle) -> torch.Tensor:
    """Expert outputs back into received order (a unit-weight top_k = 1
    combine: an exact copy of each row)."""
    return api.combine_weighted(y_grouped, handle.recv_flat_to_row, None, status=handle.status)


def combine_recv(back_rows: torch.Tensor, handle: EPHandle, weights: torch.Tensor,
                 validate: bool = False) -> torch.Tensor:
    """fused_weighted_restore of the rows returned in send order."""
    return api.combine_weighted(back_rows, handle.send_flat_to_row, weights,
                                row_to_flat=handle.send_row_to_flat, validate=validate,
                                status=handle.status)


def ep_dispatch(x: torch.Tensor, topk_idx: torch.Tensor, num_experts: int, align: int = 1,
                group=None, status: torch.Tensor | None = None):
    """Dispatch across the ranks of `group` (one GPU each): returns this
    rank's expert-grouped rows for its local experts and the handle.  Two
    all-to-alls (counts, rows) and one device-to-host copy (the splits)."""
    ep_size = dist.get_world_size(group)
    st = status if status is not None else api.new_status(x.device)
    send, lay, r2f, f2r, cm = dispatch_send(x, topk_idx, num_experts, ep_size, st)
    plan = split_plan(cm, group)
    recv = torch.empty(sum(plan.output_splits), x.shape[1], dtype=x.dtype, device=x.device)
    dist.all_to_all_single(recv, send[:sum(plan.input_splits)], plan.output_splits,
                           plan.input_splits, group=group)
    grouped, rlay, rr2f, rf2r = dispatch_recv(recv, plan, align, st)
    return grouped, EPHandle(lay, r2f, f2r, plan, rlay, rr2f, rf2r, st)


def ep_combine(y_grouped: torch.Tensor, handle: EPHandle, weights: torch.Tensor, group=None,
               validate: bool = False) -> torch.Tensor:
    """Combine across the ranks of `group`: the expert outputs go back to
    their source ranks (one all-to-all) and are restored there."""
    back = combine_send(y_grouped, handle)
    plan = handle.plan
    A = handle.send_row_to_flat.shape[0]
    returned = torch.empty(A, y_grouped.shape[1], dtype=y_grouped.dtype, device=y_grouped.device)
    dist.all_to_all_single(returned[:sum(plan.input_splits)], back, plan.input_splits,
                           plan.output_splits, group=group)
    return combine_recv(returned, handle, weights, validate)


# ------------------------------------- the payload without a send buffer ---
#
# The fused form: every rank stores its rows straight into the receive
# buffers of the ranks that own their experts (moe_permute_to_ranks), and
# gathers the expert outputs straight from them (moe_combine_from_ranks).
# The buffers are reached through a table of addresses, one per rank --
# across GPUs, the peer addresses of buffers every rank has mapped (e.g. with
# CUDA IPC or symmetric memory; the mapping itself is the caller's).  Only
# the per-expert counts are exchanged (an all-gather of [E] per rank); the
# rows cross the interconnect once, inside the kernels.  The caller puts a
# barrier between the dispatch and the experts' reads of the buffers, and
# between the experts' writes and the combine.


def rank_bases(all_counts: torch.Tensor, rank: int, align: int = 1,
               status: torch.Tensor | None = None):
    """From the per-expert counts of every source rank ([ep_size, E] int32 on
    the device, row s = rank s's tokens_per_expert): (dest_base [E] -- the
    row where `rank`'s rows of expert e start in e's owner's buffer --,
    own_offsets [E_local + 1] -- the padded group starts in `rank`'s own
    buffer --, own_counts [E_local] -- the real rows of each of its groups),
    computed by the library's moe_rank_bases kernel."""
    dest_base, own_off, own_cnt, _ = api.rank_bases(all_counts.to(torch.int32).contiguous(), rank,
                                                    align, status=status)
    return dest_base, own_off, own_cnt


def direct_receive_rows(all_counts: torch.Tensor, align: int = 1,
                        status: torch.Tensor | None = None) -> int:
    """Rows every rank's receive buffer needs for this routing (the largest
    padded total over the ranks, from moe_rank_bases).  One device-to-host
    copy: the host sizes the buffers with it."""
    _, _, _, max_rows = api.rank_bases(all_counts.to(torch.int32).contiguous(), 0, align,
                                       status=status)
    return int(max_rows.item())


def gather_counts(tokens_per_expert: torch.Tensor, group=None) -> torch.Tensor:
    """ONE all-gather of every rank's per-expert counts [E]: all_counts
    [ep_size, E] int32, row s = rank s's counts."""
    R = dist.get_world_size(group)
    E = tokens_per_expert.numel()
    all_counts = torch.empty(R, E, dtype=torch.int32, device=tokens_per_expert.device)
    dist.all_gather_into_tensor(all_counts.view(-1),
                                tokens_per_expert.to(torch.int32).contiguous().view(-1),
                                group=group)
    return all_counts


def direct_plan(tokens_per_expert: torch.Tensor, group=None, align: int = 1,
                status: torch.Tensor | None = None):
    """The metadata of the direct dispatch: the all-gather of the per-expert
    counts (gather_counts), then this rank's row bases on the device
    (rank_bases).  Returns (all_counts [ep_size, E], dest_base, own_offsets,
    own_counts)."""
    all_counts = gather_counts(tokens_per_expert, group)
    return (all_counts,) + rank_bases(all_counts, dist.get_rank(group), align, status)


@dataclasses.dataclass
class DirectHandle:
    layout: api.Layout            # this rank's tokens, one source block
    flat_to_row: torch.Tensor     # [T, K]: row in the buffer of each slot's expert rank
    own_offsets: torch.Tensor     # [E_local + 1]: this rank's groups in its own buffer
    own_counts: torch.Tensor      # [E_local]
    status: torch.Tensor


def ep_dispatch_direct(x: torch.Tensor, topk_idx: torch.Tensor, num_experts: int,
                       dest_table: torch.Tensor, dest_cap: int, align: int = 1, group=None,
                       status: torch.Tensor | None = None,
                       claims_table: torch.Tensor | None = None) -> DirectHandle:
    """Dispatch into the receive buffers listed in dest_table (one address
    per rank of `group`, each buffer [dest_cap, H] bf16).  One all-gather of
    the per-expert counts; the rows go out inside the permute.  With
    claims_table (one int32 [dest_cap] array address per rank, mapped like
    the buffers) the rows' claims are recorded for the combine's check."""
    rank = dist.get_rank(group)
    st = status if status is not None else api.new_status(x.device)
    lay = api.dispatch_layout(topk_idx, num_experts, 1, 1, status=st)
    _, dest_base, own_off, own_cnt = direct_plan(lay.tokens_per_expert, group, align, st)
    f2r = api.permute_to_ranks(x, topk_idx, lay, dest_base, dest_table, dest_cap, rank, own_off,
                               own_cnt, claims_table=claims_table, status=st)
    return DirectHandle(lay, f2r, own_off, own_cnt, st)


def ep_combine_direct(rows_table: torch.Tensor, N_cap: int, H: int, handle: DirectHandle,
                      topk_idx: torch.Tensor, weights: torch.Tensor,
                      claims_table: torch.Tensor | None = None, group=None) -> torch.Tensor:
    """fused_weighted_restore of this rank's tokens, each slot read from the
    expert-output buffer of its expert's rank (rows_table: one address per
    rank); with the dispatch's claims_table, the coverage check."""
    return api.combine_from_ranks(rows_table, N_cap, H, handle.flat_to_row, topk_idx,
                                  handle.layout.E, weights, claims_table=claims_table,
                                  rank=dist.get_rank(group) if claims_table is not None else 0,
                                  status=handle.status)
