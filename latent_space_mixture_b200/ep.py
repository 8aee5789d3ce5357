"""Expert parallelism of the LatentMoE layer: the plan and the exchange of the
latent rows between ranks ("NVIDIA Nemotron 3: Efficient and Open
Intelligence", section 三: routed experts run on the l-wide latent rows, so
an expert-parallel exchange moves l instead of d values per routed row;
"Nemotron-3 Super 精读报告" section 6.5: 64-way expert parallelism).

Layout.  The N experts are split into P contiguous ranges, rank r owning
experts [r N / P, (r + 1) N / P).  Each rank routes its own tokens; its
routed rows in expert order (expert, then token, then slot: the order of the
forward's segments) are therefore already grouped by destination rank, so a
rank sends the contiguous slice of its expert-order rows that belongs to each
destination.  A rank receives, from every source in rank order, the rows for
its experts, each source's rows in expert order; the local grouped GEMMs want
them grouped by expert, so the receiver re-sorts them (expert, then source,
then the source's order).  The combine runs the same steps backwards: the
expert outputs go back to source order, through the reverse all-to-all, and
arrive in the sender's expert order, where the weighted sum per token runs.

This module holds no arithmetic of the layer: it computes counts,
permutations and split sizes, and moves rows with
torch.distributed.all_to_all_single (NCCL on GPUs, gloo on CPU).  On GPUs,
`forward` runs one rank's layer with the library's expert-parallel calls:
lmoe_forward_dispatch (the latent rows in expert order), the all-to-all,
lmoe_permute_rows (into local expert order), lmoe_experts_forward (the
rank's shard of experts), the way back, and lmoe_forward_combine.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import torch
import torch.distributed as dist

__all__ = ["expert_range", "EPPlan", "plan", "plan_from_counts", "dispatch", "combine",
           "forward"]


def expert_range(N: int, P: int, rank: int):
    """[first, last) experts of `rank` (N a multiple of P)."""
    if N % P:
        raise ValueError("the expert count must be a multiple of the ranks")
    per = N // P
    return rank * per, (rank + 1) * per


@dataclass
class EPPlan:
    """The exchange of one forward on one rank.

    send_counts[d]   rows this rank sends to rank d (its expert-order rows of
                     d's experts, contiguous);
    recv_counts[s]   rows this rank receives from rank s;
    recv_counts_e    [P][N/P] rows from source s for local expert j;
    local_order      [R_in]: position in the received buffer of the i-th row
                     in local expert order (expert, source, source order);
    local_counts     [N/P] rows per local expert.
    """
    send_counts: List[int]
    recv_counts: List[int]
    recv_counts_e: torch.Tensor
    local_order: torch.Tensor
    local_counts: torch.Tensor


def plan(counts: torch.Tensor, group: Optional[dist.ProcessGroup] = None) -> EPPlan:
    """Exchange plan from this rank's routed rows per expert (counts [N], int,
    on the host): the counts of every (source, local expert) pair are
    exchanged first (one all-to-all of P x N/P integers)."""
    P = dist.get_world_size(group)
    N = counts.numel()
    per = N // P
    if N % P:
        raise ValueError("the expert count must be a multiple of the ranks")
    c = counts.to(torch.int64).reshape(P, per)          # [dest][local expert of dest]
    recv_e = torch.empty_like(c)                         # [source][my local expert]
    dist.all_to_all_single(recv_e.reshape(-1), c.reshape(-1).contiguous(), group=group)
    return plan_from_counts(c, recv_e)


def plan_from_counts(c: torch.Tensor, recv_e: torch.Tensor) -> EPPlan:
    """The plan of one rank from its own rows per (destination, local expert
    of the destination), c [P][N/P], and the rows every source sends for
    this rank's local experts, recv_e [P][N/P] (host int64 tensors)."""
    P, per = c.shape
    send_counts = c.sum(dim=1).tolist()
    recv_counts = recv_e.sum(dim=1).tolist()
    # received buffer: source-major, each source's rows by local expert
    src_base = torch.zeros(P + 1, dtype=torch.int64)
    src_base[1:] = torch.cumsum(recv_e.sum(dim=1), 0)
    within = torch.zeros_like(recv_e)                    # start of (s, j) within source s
    within[:, 1:] = torch.cumsum(recv_e, dim=1)[:, :-1]
    order = []
    for j in range(per):
        for s in range(P):
            n = int(recv_e[s, j])
            if n:
                start = int(src_base[s] + within[s, j])
                order.append(torch.arange(start, start + n, dtype=torch.int64))
    local_order = torch.cat(order) if order else torch.zeros(0, dtype=torch.int64)
    return EPPlan(send_counts, recv_counts, recv_e, local_order, recv_e.sum(dim=0))


def dispatch(rows: torch.Tensor, p: EPPlan, group: Optional[dist.ProcessGroup] = None):
    """Expert-order rows of this rank [sum(send_counts)][l] -> the rows of the
    local experts in local expert order [sum(recv_counts)][l]."""
    recv = rows.new_empty((sum(p.recv_counts),) + tuple(rows.shape[1:]))
    dist.all_to_all_single(recv, rows.contiguous(), p.recv_counts, p.send_counts, group=group)
    return recv.index_select(0, p.local_order.to(recv.device))


def combine(rows: torch.Tensor, p: EPPlan, group: Optional[dist.ProcessGroup] = None):
    """Outputs of the local experts in local expert order -> this rank's
    routed rows in its expert order (the inverse of dispatch)."""
    back = torch.empty_like(rows)
    back.index_copy_(0, p.local_order.to(rows.device), rows)
    out = rows.new_empty((sum(p.send_counts),) + tuple(rows.shape[1:]))
    dist.all_to_all_single(out, back.contiguous(), p.send_counts, p.recv_counts, group=group)
    return out


def forward(layer, shard, x: torch.Tensor, group: Optional[dist.ProcessGroup] = None):
    """One rank's expert-parallel forward on GPUs: `layer` a LatentMoE built
    with ep_dense=True (router, projections, shared expert), `shard` the
    ExpertShard of this rank's expert range (expert_range), x [T][d] this
    rank's tokens.  The exchanged rows are l wide.  Returns y [T][d]."""
    from .layer import lmoe_permute_rows
    rows, counts = layer.dispatch(x)
    p = plan(counts.cpu(), group)
    recv = rows.new_empty((sum(p.recv_counts), rows.shape[1]))
    dist.all_to_all_single(recv, rows, p.recv_counts, p.send_counts, group=group)
    order = p.local_order.to(torch.int32).to(rows.device)
    local = lmoe_permute_rows(recv, order, scatter=False)
    out = shard.forward(local, p.local_counts.to(torch.int32).to(rows.device))
    back = lmoe_permute_rows(out, order, scatter=True, out_rows=recv.shape[0])
    got = torch.empty_like(rows)
    dist.all_to_all_single(got, back, p.send_counts, p.recv_counts, group=group)
    return layer.combine(got)
