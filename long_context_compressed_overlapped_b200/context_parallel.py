"""Context parallelism for a compressed-attention decode layer.

"Paper Breakdown: DeepSeek-V4", infrastructure table: "2-Stage Context
Parallel" for compressed attention.  The page names the technique and gives
no steps; the reading taken here splits a layer's compressed cache by entry
range over the ranks of a process group and takes one decode step in two
exchange stages:

  stage 1 (CSA only): every rank scores its own shard with the lightning
      indexer and keeps its top-k (local rows and their scores); the ranks
      all-gather these candidates and each merges them into the global
      top-k.  Every entry of the global top-k is in the top-k of its own
      shard, so the merge equals the top-k over the whole cache.
  stage 2: every rank attends over its own part of the keys (its selected
      rows for CSA, its visible rows for HCA; the window on one rank only)
      and writes an unnormalised share (max logit, sum of weights, weighted
      mean per head); the ranks all-gather the shares and each combines them
      with the sink and rotates the output back by -t.

The compute steps are the library's kernels (`GpuOps`: indexer_topk with
entry_base and sel_scores, cp_topk_merge, compressed_attn_decode with
partial_out, cp_attn_merge); the exchanges are `torch.distributed`
all-gathers (NCCL between GPUs).  `CPDecodeLayer` takes the ops and the
exchange as arguments, so the same schedule runs on any backend that
implements them.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Protocol, Sequence

import torch
import torch.distributed as dist

from . import api


def shard_ranges(n_entries: int, world: int) -> list[tuple[int, int]]:
    """(first global entry, entry count) of each rank's shard: contiguous
    ranges in rank order, the first n_entries % world ranks one longer."""
    if world < 1 or n_entries < 0:
        raise ValueError("shard_ranges: world >= 1 and n_entries >= 0")
    base, extra = divmod(n_entries, world)
    out, start = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((start, n))
        start += n
    return out


class Exchange(Protocol):
    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        """[world, *t.shape]: every rank's t in rank order."""


class DistExchange:
    """All-gathers over a torch.distributed process group (NCCL for CUDA
    tensors, gloo for host tensors)."""

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group)

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        t = t.contiguous()
        out = torch.empty(self.world * t.numel(), dtype=t.dtype, device=t.device)
        # flat buffers: the form every backend's all-gather into one tensor takes
        dist.all_gather_into_tensor(out, t.view(-1), group=self.group)
        return out.view((self.world,) + tuple(t.shape))


class Ops(Protocol):
    def local_topk(self, L: "Shard", q_pos: torch.Tensor, k: int): ...
    def topk_merge(self, cand_idx, cand_scores, bases: Sequence[int], rank: int): ...
    def local_share(self, L: "Shard", pos: torch.Tensor, idx_local, skip_window: bool): ...
    def merge(self, shares, L: "Shard", pos: torch.Tensor): ...


@dataclass
class Shard:
    """One rank's part of a decode layer: its cache shard (global entries
    entry_base .. entry_base + N - 1) and the inputs every rank holds."""
    kind: str                       # "csa" or "hca"
    entry_base: int
    q: torch.Tensor                 # [B, H, d] raw new queries
    kv: torch.Tensor                # [B, N, d] final rows of the shard (or FP8 KV rows, uint8)
    win: torch.Tensor               # [B, w, d] window ring
    sinks: torch.Tensor             # [H]
    m: int
    rope_dims: int
    q_gain: torch.Tensor | None = None
    qI: torch.Tensor | None = None  # CSA: [B, HI, dI]
    wI: torch.Tensor | None = None  # CSA: [B, HI]
    kI: torch.Tensor | None = None  # CSA: [B, N, dI] shard of the indexer keys
    kI_scale: torch.Tensor | None = None
    k: int = 0


class GpuOps:
    """The library's kernels for the four compute steps."""

    def local_topk(self, L: Shard, pos, k):
        B = L.q.shape[0]
        sel = torch.empty(B, 1, k, dtype=torch.float32, device=L.q.device)
        idx = api.indexer_topk(L.qI[:, None], L.wI[:, None], L.kI, pos[:, None], L.m, k, kI_scale=L.kI_scale,
                               sel_scores=sel, entry_base=L.entry_base)
        return idx[:, 0], sel[:, 0]

    def topk_merge(self, cand_idx, cand_scores, bases, rank):
        return api.cp_topk_merge(cand_idx, cand_scores, bases, rank)[1]

    def local_share(self, L: Shard, pos, idx_local, skip_window):
        B, H, d = L.q.shape
        share = torch.empty(B, api.cp_partial_floats(H, d), dtype=torch.float32, device=L.q.device)
        kw = dict(k=L.k, idx_in=idx_local) if L.kind == "csa" else {}
        return api.compressed_attn_decode(L.kind, L.q, pos, L.kv, L.win, L.sinks, m=L.m, rope_dims=L.rope_dims,
                                          q_gain=L.q_gain, entry_base=L.entry_base, partial_out=share,
                                          skip_window=skip_window, **kw)

    def merge(self, shares, L: Shard, pos):
        B, H, d = L.q.shape
        return api.cp_attn_merge(shares, L.sinks, pos, H=H, d=d, rope_dims=L.rope_dims, dtype=L.q.dtype)


class CPDecodeLayer:
    """One rank's schedule of a context-parallel decode step of one layer.

    bases: every rank's first global entry (the same list on all ranks);
    window_rank: the rank that attends the window (the one holding the
    newest entries is the natural choice)."""

    def __init__(self, rank: int, bases: Sequence[int], exchange: Exchange, ops: Ops | None = None,
                 window_rank: int | None = None):
        self.rank = rank
        self.bases = [int(b) for b in bases]
        self.exchange = exchange
        self.ops = ops if ops is not None else GpuOps()
        self.window_rank = len(self.bases) - 1 if window_rank is None else window_rank
        if not 0 <= rank < len(self.bases) or not 0 <= self.window_rank < len(self.bases):
            raise ValueError("CPDecodeLayer: rank and window_rank must name ranks of bases")

    # The four stages, callable one by one (a caller that runs several ranks'
    # shards in one process exchanges between them itself).
    def local_candidates(self, L: Shard, pos: torch.Tensor):
        """Stage 1, local: this shard's top-k (local rows [B, k], scores [B, k])."""
        self._check(L)
        return self.ops.local_topk(L, pos, L.k)

    def merge_candidates(self, cand_idx: torch.Tensor, cand_scores: torch.Tensor) -> torch.Tensor:
        """Stage 1, after the exchange: this rank's local rows of the global top-k [B, k]."""
        return self.ops.topk_merge(cand_idx, cand_scores, self.bases, self.rank)

    def local_share(self, L: Shard, pos: torch.Tensor, idx_local) -> torch.Tensor:
        """Stage 2, local: this rank's unnormalised share [B, 2H + H*d]."""
        self._check(L)
        return self.ops.local_share(L, pos, idx_local, skip_window=self.rank != self.window_rank)

    def merge_shares(self, shares: torch.Tensor, L: Shard, pos: torch.Tensor) -> torch.Tensor:
        """Stage 2, after the exchange: the layer output [B, H, d]."""
        return self.ops.merge(shares, L, pos)

    def __call__(self, L: Shard, pos: torch.Tensor) -> torch.Tensor:
        idx_local = None
        if L.kind == "csa":
            idx_l, sc_l = self.local_candidates(L, pos)
            idx_local = self.merge_candidates(self.exchange.all_gather(idx_l), self.exchange.all_gather(sc_l))
        share = self.local_share(L, pos, idx_local)
        return self.merge_shares(self.exchange.all_gather(share), L, pos)

    def _check(self, L: Shard) -> None:
        if L.entry_base != self.bases[self.rank]:
            raise ValueError("CPDecodeLayer: the shard's entry_base is not this rank's base")
