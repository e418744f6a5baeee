"""Expert parallelism: the host-side dispatch and combine of the MoE block over ranks.

The model pages shard the experts over devices: the Inferentia2 build places 16 experts on
each of 8 NeuronCores ("Gemma-4 26B-A4B (MoE) on AWS Inferentia2", "How it works"), the
Tenstorrent build runs TP4 + EP4 ("Gemma-4-26B-A4B-it - Tenstorrent Blackhole", "Model /
precision"), and the inference recipe lists expert-parallel strategies ("Gemma 4 26B-A4B
IT", `compatible_strategies`).  Here every rank keeps its own batch of tokens (data
parallel), owns E / world experts, and routes and sorts its tokens with the full router.
One exchange pair moves the work:

  dispatch  the routed rows (xn_moe of each (token, slot) pair, in the rank's expert-sorted
            order) go to the rank that owns the pair's expert (the routing weights stay
            with the source, which applies them in its combine).  In
            sorted order the pairs of one destination are contiguous (owners hold
            consecutive experts), so the send list is the sorted rows cut at the owners'
            boundaries; the per-expert counts travel first, so every receiver knows how its
            rows are laid out before any row arrives.
  compute   the receiver orders its rows expert-major (stable: by expert, then source
            rank, then position), runs its experts on them and returns each row's
            unweighted expert output in the order it received the row.
  combine   the returned rows land at their pairs' sorted positions, and the block's usual
            combine (slot order j = 0..k-1, routing weights in fp32) finishes the branch.

Every transfer is a torch.distributed all_to_all (NCCL over NVLink on GPUs, gloo on the
host): remote rows land in local memory before any kernel reads them; no kernel is given
another rank's memory.  This module holds the bookkeeping only (counts, offsets and the
permutations between the orders above); the arithmetic on the rows is the caller's
(`compute`), so the same exchange drives the library's expert kernels on a GPU and the
oracle in the CPU tests.
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist


@dataclasses.dataclass(frozen=True)
class ExpertPartition:
    """E experts over `world` ranks: rank r owns experts [r * E / world, (r + 1) * E / world)."""
    num_experts: int
    world: int

    def __post_init__(self):
        if self.world < 1 or self.num_experts % self.world:
            raise ValueError("the experts must divide evenly over the ranks")

    @property
    def local(self) -> int:
        return self.num_experts // self.world

    def owner(self, e):
        return e // self.local

    def first(self, rank: int) -> int:
        return rank * self.local


def send_counts(offsets: torch.Tensor, part: ExpertPartition) -> torch.Tensor:
    """Rows for each destination rank, from the expert offsets [E + 1] of the rank's own
    sorted pairs: destination d gets sorted positions [offsets[d * El], offsets[(d+1) * El])."""
    cut = offsets[torch.arange(0, part.num_experts + 1, part.local)]
    return (cut[1:] - cut[:-1]).to(torch.int64)


def local_counts(offsets: torch.Tensor, part: ExpertPartition) -> torch.Tensor:
    """Per-expert counts of this rank's pairs, as [world][E_local]: row d holds the counts
    of destination d's experts (what d needs to lay out the rows it receives from us)."""
    c = (offsets[1:] - offsets[:-1]).to(torch.int64)
    return c.view(part.world, part.local)


def receive_layout(recv_counts: torch.Tensor):
    """From the counts every source sent for our experts ([world][E_local]: row s = source
    s), the layout of the received rows: they arrive grouped by source, and within a
    source grouped by expert.  Returns (local_offsets [E_local + 1], order) where order[q]
    is the received-row index of the q-th row in expert-major order (by expert, then source,
    then arrival position): the stable sort of the received rows by expert."""
    world, el = recv_counts.shape
    src_rows = recv_counts.sum(dim=1)                         # rows from each source
    src_start = torch.cumsum(src_rows, 0) - src_rows          # first received row of each source
    # first received row of (source s, expert e): the source's start + its earlier experts
    within = torch.cumsum(recv_counts, dim=1) - recv_counts
    start = src_start[:, None] + within                       # [world][E_local]
    per_expert = recv_counts.sum(dim=0)                       # [E_local]
    local_offsets = torch.zeros(el + 1, dtype=torch.int64)
    local_offsets[1:] = torch.cumsum(per_expert, 0)
    pieces = []
    for e in range(el):
        for s in range(world):
            n = int(recv_counts[s, e])
            if n:
                pieces.append(torch.arange(int(start[s, e]), int(start[s, e]) + n, dtype=torch.int64))
    order = torch.cat(pieces) if pieces else torch.zeros(0, dtype=torch.int64)
    return local_offsets, order


def _all_to_all_rows(send: torch.Tensor, send_counts_: torch.Tensor, recv_counts_: torch.Tensor,
                     group=None) -> torch.Tensor:
    """All-to-all of row blocks of varying sizes (the rows of one destination contiguous)."""
    recv = send.new_empty((int(recv_counts_.sum()),) + tuple(send.shape[1:]))
    dist.all_to_all_single(recv, send.contiguous(), output_split_sizes=recv_counts_.tolist(),
                           input_split_sizes=send_counts_.tolist(), group=group)
    return recv


def ep_moe_forward(rows_sorted: torch.Tensor, offsets: torch.Tensor, part: ExpertPartition,
                   compute, group=None) -> torch.Tensor:
    """One dispatch / compute / return over the ranks.

    rows_sorted [T*k][H]: this rank's routed rows in its expert-sorted order (row q is pair
    sorted_src[q]'s token row); offsets [E + 1]: the expert offsets of that order.
    compute(expert_rows, local_offsets) -> outputs: runs this rank's E_local experts on the
    received rows in expert-major order (expert e's rows are
    [local_offsets[e], local_offsets[e + 1])) and returns one output row per input row.
    Returns [T*k][...]: the output of each of this rank's pairs, in its sorted order (the
    caller's combine applies the routing weights in slot order).
    """
    offsets = offsets.to(torch.int64)
    s_counts = send_counts(offsets, part)
    # per-expert counts first: receivers lay out rows before the rows arrive
    mine = local_counts(offsets, part)                        # [world][E_local] by destination
    theirs = torch.empty_like(mine)
    dist.all_to_all_single(theirs, mine.contiguous(), group=group)  # row s: source s's counts
    r_counts = theirs.sum(dim=1)
    recv = _all_to_all_rows(rows_sorted, s_counts, r_counts, group)
    local_offsets, order = receive_layout(theirs)
    out_sorted = compute(recv[order], local_offsets)          # expert-major
    back = out_sorted.new_empty((recv.shape[0],) + tuple(out_sorted.shape[1:]))
    back[order] = out_sorted                                  # received order again
    return _all_to_all_rows(back, r_counts, s_counts, group)  # our pairs, in our sorted order
