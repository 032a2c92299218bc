"""Context-parallel decode of long sequences: G ranks (or G logical shards on
one device) each own a contiguous, page-aligned range of positions of every
sequence, and one decode step computes exactly what the unsharded step
computes.

The split is the multi-GPU plan of the scope table (the pages name DCP only as
a runtime concern: page "DeepSeek V4 1-Flash 架构拆解…" (blog.zulogic.cn),
section 10 and section 13 "DCP 稀疏索引一致性"). Per step, for one query token
per sequence:
  1. each shard scores its own positions and keeps its top-k with the scores
     (csa2_indexer_topk_scores), as global positions;
  2. the (score, position) candidates of all shards are all-gathered: k x 8 B
     per query row and shard;
  3. every shard selects the global top-k from the candidates
     (csa2_topk_merge; a shard's own top-k holds all of its positions that are
     in the global top-k, and the tie rule is the same) and keeps the entries
     it owns, as local positions;
  4. each shard attends over its owned entries; the shard holding the newest
     positions also attends over the 128-row window (csa2_sparse_attn_decode,
     without a window elsewhere);
  5. the normalised partial results (o, lse) are all-gathered: 16 x 577 floats
     per query row and shard;
  6. one softmax over the union (csa2_lse_merge).
Sharing the page table: shard g reads the same physical pages as the whole
sequence through the columns of the page table for its range, so no cache is
copied to form the shards.

The exchange is torch.distributed.all_gather (NCCL between GPUs);
no data-path step uses TMA multicast or a library kernel on a peer's memory.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional, Tuple

import torch

PAGE = 64


@dataclasses.dataclass
class Shard:
    """Shard g of G: positions [lo, hi) of every sequence (hi = the longest
    sequence for the last shard), seen through its own page-table columns."""
    g: int
    G: int
    lo: int
    hi: int
    page_table: torch.Tensor      # [B, (hi - lo) / 64] int32: columns lo/64 .. hi/64 of the full table
    seq_lens: torch.Tensor        # [B] int32: positions of each sequence inside the shard

    @property
    def has_window(self) -> bool:
        """The last shard holds every sequence's newest positions, so it
        attends over the window rows."""
        return self.g == self.G - 1


def shard_bounds(max_len: int, G: int, g: int) -> Tuple[int, int]:
    """Page-aligned contiguous split of [0, max_len) into G ranges; the last
    range ends at max_len."""
    pages = -(-max_len // PAGE)
    p0 = pages * g // G
    p1 = pages * (g + 1) // G
    return p0 * PAGE, (max_len if g == G - 1 else p1 * PAGE)


def make_shard(page_table: torch.Tensor, seq_lens: torch.Tensor, G: int, g: int) -> Shard:
    """Shard g of a paged cache. Every sequence must be long enough to reach
    the last shard (its newest position is where the query sits)."""
    max_len = int(page_table.shape[1]) * PAGE
    lo, hi = shard_bounds(max_len, G, g)
    lens = seq_lens.to(torch.int64)
    if g == G - 1 and lo > 0 and bool((lens - lo < 128).any()):
        # the last shard attends over the window: its 128 rows must be its own positions
        raise ValueError("every sequence must hold at least 128 positions in the last shard")
    cols = page_table[:, lo // PAGE: -(-hi // PAGE)].contiguous()
    local = torch.clamp(torch.minimum(lens, torch.full_like(lens, hi)) - lo, min=0).to(torch.int32)
    return Shard(g, G, lo, hi, cols, local.contiguous())


class GpuOps:
    """The per-shard steps through the CUDA library."""

    def __init__(self, lib, cache, k: int, softmax_scale: float):
        self.lib, self.cache, self.k, self.scale = lib, cache, k, softmax_scale

    def local_candidates(self, shard: Shard, q_idx, w) -> Tuple[torch.Tensor, torch.Tensor]:
        idx, sc = self.lib.indexer_topk_scores(q_idx, w, self.cache, shard.page_table, shard.seq_lens, self.k)
        gidx = torch.where(idx >= 0, idx + shard.lo, idx)
        B, Sq = q_idx.shape[0], q_idx.shape[1]
        return sc.view(B * Sq, self.k), gidx.view(B * Sq, self.k)

    def own_entries(self, shard: Shard, all_scores, all_idx) -> torch.Tensor:
        _, local = self.lib.topk_merge(all_scores, all_idx, self.k, shard.lo, shard.hi, want_global=False,
                                       want_local=True)
        return local

    def attend(self, shard: Shard, q, swa, local_idx) -> Tuple[torch.Tensor, torch.Tensor]:
        B, Sq = q.shape[0], q.shape[1]
        idx = local_idx.view(B, Sq, self.k)
        o, lse = self.lib.sparse_attn_decode(q, self.cache, shard.page_table, shard.seq_lens, idx,
                                             swa if shard.has_window else None, self.scale)
        return o.view(B * Sq, 16, 576), lse.view(B * Sq, 16)

    def combine(self, all_o, all_lse) -> Tuple[torch.Tensor, torch.Tensor]:
        return self.lib.lse_merge(all_o, all_lse)


def decode_step(shard: Shard, ops, q, q_idx, w, swa,
                all_gather: Callable[[torch.Tensor], torch.Tensor]) -> Tuple[torch.Tensor, torch.Tensor]:
    """One context-parallel decode step on this shard. all_gather(t) returns
    the G shards' tensors stacked in shard order ([G, *t.shape]). Every shard
    returns the same (o [R, 16, 576], lse [R, 16])."""
    sc, gi = ops.local_candidates(shard, q_idx, w)
    all_sc, all_gi = all_gather(sc), all_gather(gi)
    local = ops.own_entries(shard, all_sc, all_gi)
    o, lse = ops.attend(shard, q, swa, local)
    return ops.combine(all_gather(o), all_gather(lse))


def dist_all_gather(group=None) -> Callable[[torch.Tensor], torch.Tensor]:
    """all_gather over a torch.distributed process group (NCCL between GPUs,
    gloo on CPU), stacked in rank order."""
    import torch.distributed as dist

    def gather(t: torch.Tensor) -> torch.Tensor:
        world = dist.get_world_size(group)
        parts = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t.contiguous(), group=group)
        return torch.stack(parts)

    return gather


def decode_step_in_process(shards: List[Shard], ops_for: Callable[[Shard], object], q, q_idx, w, swa
                           ) -> Tuple[torch.Tensor, torch.Tensor]:
    """All G shards on one device, phase by phase, with the all-gathers done
    by stacking: the same arithmetic as G ranks."""
    ops = [ops_for(s) for s in shards]
    cands = [op.local_candidates(s, q_idx, w) for op, s in zip(ops, shards)]
    all_sc = torch.stack([c[0] for c in cands])
    all_gi = torch.stack([c[1] for c in cands])
    parts = [op.attend(s, q, swa, op.own_entries(s, all_sc, all_gi)) for op, s in zip(ops, shards)]
    return ops[0].combine(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
