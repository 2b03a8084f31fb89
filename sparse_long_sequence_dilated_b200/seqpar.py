"""Sequence-parallel dilated attention forward over ranks (one GPU per rank).

LongNet splits the sequence across devices (the gptget.net summary of arXiv
2307.02486, "方法详解" bullet 5, and the abstract's second contribution):
with world ranks, rank g holds positions [g L, (g + 1) L), L = N / world.

* A pattern whose segments fit in a block (w <= L, L a multiple of w) is
  computed where the block lives: nothing crosses ranks.
* A pattern with w > L has segments spanning min(w, N) / L ranks. Inside a
  block, head h keeps the rows (h mod r) + m r (the block start is a
  multiple of r), so every rank sends just those L / r rows of k and v; the
  ranks of the segment all-gather them in rank order and each rank attends
  its own kept query rows to the gathered dilated sequence, causal with its
  block's offset in that sequence.

Every pattern's result for a row ends up on the rank that owns the row, so
the cross-pattern merge stays local. The all-gathers run with
torch.distributed (NCCL on GPUs, gloo on the CPU) inside each segment's run
of consecutive ranks (one set of subgroups per segment size); the kernels
are the library's (dilattn_pack_dilated, dilattn_fwd_seqpar). This module
holds only the bookkeeping.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

BM = 128  # rows per tile: a rank's dilated block must be whole tiles


@dataclasses.dataclass(frozen=True)
class PatternPlan:
    index: int
    w: int
    r: int
    spans: bool          # segments span several ranks
    ranks: int = 1       # ranks per segment (spans only)
    rank_rows: int = 0   # dilated rows each rank contributes per head (spans only)

    def segment_ranks(self, rank: int) -> List[int]:
        """The ranks whose blocks form this rank's segment, in sequence order."""
        if not self.spans:
            return [rank]
        first = (rank // self.ranks) * self.ranks
        return list(range(first, first + self.ranks))

    def tile_offset(self, rank: int) -> int:
        """Key tile of the gathered sequence where this rank's query tiles start."""
        return (rank % self.ranks) * (self.rank_rows // BM) if self.spans else 0


def plan(N: int, world: int, patterns: Sequence[Tuple[int, int]]) -> List[PatternPlan]:
    """Which patterns stay local and how spanning ones are gathered; raises
    ValueError for splits the kernels do not take (the same checks as
    dilattn_fwd_seqpar)."""
    if world < 1 or N % world != 0:
        raise ValueError("N must be a multiple of the number of ranks")
    L = N // world
    out = []
    for i, (w, r) in enumerate(patterns):
        if w <= L:
            if L % w != 0:
                raise ValueError(f"pattern {i}: the block length {L} is not a multiple of w = {w}")
            out.append(PatternPlan(i, w, r, False))
            continue
        span = min(w, N)
        if span % L != 0 or (w < N and N % w != 0):
            raise ValueError(f"pattern {i}: segments of w = {w} do not cover whole blocks of {L}")
        if L % r != 0 or (L // r) % BM != 0:
            raise ValueError(f"pattern {i}: L / r = {L} / {r} must be a whole number of {BM}-row tiles")
        out.append(PatternPlan(i, w, r, True, span // L, L // r))
    return out


def packed_positions(p: PatternPlan, L: int, rank: int, h: int):
    """Global positions of the rows rank `rank` sends for head h (the rows
    dilattn_pack_dilated extracts): rank L + (h mod r) + m r, m < L / r."""
    return [rank * L + (h % p.r) + m * p.r for m in range(L // p.r)]


# subgroups of the default group, one set per segment size: ranks -> (the default
# group they were made from, this rank's subgroup)
_SEGMENT_GROUPS: dict = {}


def segment_group(ranks: int, world: int, group=None):
    """The process group a segment of `ranks` consecutive blocks gathers over.

    Segments tile the ranks in consecutive runs, so for the default group the
    gather runs inside this rank's run only (torch.distributed.new_subgroups,
    created once per segment size; every rank reaches them in the same order
    because every rank plans the same patterns). A segment over every rank, or
    a caller's own group, gathers over that group."""
    if ranks == world or group is not None:
        return group
    import torch.distributed as dist
    made = _SEGMENT_GROUPS.get(ranks)
    if made is None or made[0] is not dist.group.WORLD:  # none yet, or a new default group
        made = (dist.group.WORLD, dist.new_subgroups(group_size=ranks)[0])
        _SEGMENT_GROUPS[ranks] = made
    return made[1]


def forward(q, k, v, patterns, causal: bool = True, group=None, out=None, lse=None, stream=None):
    """This rank's rows of the dilated-attention forward: (out [B, L, H, d], lse [B, H, L]).

    q, k, v: this rank's block [B, L, H, d] (bf16, on its GPU). Collective:
    every rank of the group calls it with the same patterns, in the same order.
    Each spanning pattern's rows are gathered among the ranks of the segment
    (a subgroup of the default group), so a rank receives (ranks - 1) packs per
    pattern, not (world - 1)."""
    import torch
    import torch.distributed as dist

    from . import dilattn

    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    B, L, H, d = q.shape
    plans = plan(L * world, world, patterns)
    kg: List[Optional[object]] = [None] * len(plans)
    vg: List[Optional[object]] = [None] * len(plans)
    for p in plans:
        if not p.spans:
            continue
        sub = segment_group(p.ranks, world, group)
        n = p.ranks if sub is not group else world  # ranks taking part in the gather
        bufs = []
        for x in (k, v):
            send = dilattn.pack_dilated(x, p.r, stream=stream)
            # the packs concatenated along the batch dimension (the form every
            # backend takes), the same memory as [n, B, L/r, H, d] in rank order
            recv = torch.empty((n * send.shape[0],) + tuple(send.shape[1:]),
                               dtype=send.dtype, device=send.device)
            dist.all_gather_into_tensor(recv, send, group=sub)
            recv = recv.view((n,) + tuple(send.shape))
            if n == world and p.ranks < world:
                first = p.segment_ranks(rank)[0]
                recv = recv[first:first + p.ranks]
            bufs.append(recv)  # contiguous: [ranks, B, L/r, H, d]
        kg[p.index], vg[p.index] = bufs
    return dilattn.fwd_seqpar(q, k, v, patterns, rank, world, kg, vg, causal, out, lse, stream)
