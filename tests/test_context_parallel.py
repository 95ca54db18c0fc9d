"""Context parallelism on CPU: the two-stage schedule of
long_context_compressed_overlapped_b200.context_parallel ("Paper Breakdown:
DeepSeek-V4", infrastructure table, "2-Stage Context Parallel"), with the
compute steps written out from the oracle (tests/cp_oracle_ops.py), against
the oracle's unsharded decode layer: the global top-k must equal the
oracle's top-k over the whole cache exactly (ties to the lower entry, across
shard boundaries too) and the output must match to float64 rounding.

Two forms: ranks emulated in one process (exchanges by stacking), and real
gloo ranks (world sizes 2 and 3) exchanging through torch.distributed."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_compressed_overlapped_b200 import context_parallel as CP
from tests.cp_oracle_ops import OracleOps, make_layer, reference, shard_of

TOL = 1e-12


def _run_emulated(L, pos, ranges, ops=None, window_rank=None):
    """Every rank's stages in lockstep in one process; returns each rank's
    output and its local selection."""
    ops = ops or OracleOps()
    bases = [b for b, _ in ranges]
    layers = [CP.CPDecodeLayer(r, bases, exchange=None, ops=ops, window_rank=window_rank)
              for r in range(len(ranges))]
    shards = [shard_of(L, b, n, CP.Shard) for b, n in ranges]
    idx = [None] * len(ranges)
    if L["kind"] == "csa":
        cands = [cp.local_candidates(s, pos) for cp, s in zip(layers, shards)]
        ci = torch.stack([c[0] for c in cands])
        cs = torch.stack([c[1] for c in cands])
        idx = [cp.merge_candidates(ci, cs) for cp in layers]
    shares = torch.stack([cp.local_share(s, pos, ix) for cp, s, ix in zip(layers, shards, idx)])
    outs = [cp.merge_shares(shares, s, pos) for cp, s in zip(layers, shards)]
    return outs, idx, bases


def _global_selection(idx_local, bases):
    """The union of the ranks' local selections as global entries, sorted."""
    B, k = idx_local[0].shape
    out = []
    for b in range(B):
        g = sorted(int(bases[r] + x) for r, ix in enumerate(idx_local) for x in ix[b].tolist() if x >= 0)
        out.append(g + [-1] * (k - len(g)))
    return np.array(out)


def _check(L, pos, outs, idx_local, bases):
    ref, sel = reference(L, pos)
    for o in outs:
        err = np.abs(o.numpy() - ref).max()
        assert err <= TOL, f"output max-abs {err:.3e}"
    if sel is not None:
        assert (_global_selection(idx_local, bases) == sel).all(), "global top-k differs from the oracle's"


CASES = [
    # kind, ranges of the 64-entry cache, positions of the two sequences
    ("csa", CP.shard_ranges(64, 2), [255, 200]),
    ("csa", CP.shard_ranges(64, 3), [255, 37]),        # second sequence sees rank 0's shard only
    ("csa", [(0, 10), (10, 40), (50, 14)], [255, 3]),  # uneven shards; t < m - 1 sees nothing
    ("csa", CP.shard_ranges(64, 4), [30, 255]),        # fewer than k visible in total
    ("hca", CP.shard_ranges(64, 2), [1023, 700]),
    ("hca", CP.shard_ranges(64, 3), [1023, 15]),       # 15 = m' - 1: one entry visible
]


@pytest.mark.parametrize("kind,ranges,pos", CASES)
def test_emulated_ranks_match_unsharded_oracle(kind, ranges, pos):
    L = make_layer(kind, seed=3)
    p = torch.tensor(pos, dtype=torch.int32)
    outs, idx, bases = _run_emulated(L, p, ranges)
    _check(L, p, outs, idx, bases)


def test_window_owner_may_be_any_rank():
    L = make_layer("hca", seed=4)
    p = torch.tensor([1023, 300], dtype=torch.int32)
    for wr in range(3):
        outs, idx, bases = _run_emulated(L, p, CP.shard_ranges(64, 3), window_rank=wr)
        _check(L, p, outs, idx, bases)


def test_ties_across_shards_go_to_the_lower_entry():
    """Indexer keys of entries 5, 40 and 60 made equal to those of 20, 33 and
    2 (so their scores tie exactly, across the shard boundaries): the merge
    must keep the lower global entry, as the oracle's top-k over one cache."""
    L = make_layer("csa", seed=5, k=6, tie_pairs=[(20, 5), (33, 40), (2, 60)])
    p = torch.tensor([255, 255], dtype=torch.int32)
    outs, idx, bases = _run_emulated(L, p, CP.shard_ranges(64, 2))
    _check(L, p, outs, idx, bases)
    # all-equal keys: the first k entries win
    L["kI"][:] = L["kI"][:, :1]
    outs, idx, bases = _run_emulated(L, p, CP.shard_ranges(64, 3))
    assert (_global_selection(idx, bases) == np.arange(6)[None]).all()
    _check(L, p, outs, idx, bases)


class _TieHigh(OracleOps):
    def topk_merge(self, cand_idx, cand_scores, bases, rank):
        # planted mistake: ties to the HIGHER global entry
        R, B, k = cand_idx.shape
        out = np.full((B, k), -1, np.int64)
        for b in range(B):
            g = np.concatenate([bases[r] + cand_idx[r, b].numpy()[cand_idx[r, b].numpy() >= 0] for r in range(R)])
            s = np.concatenate([cand_scores[r, b].numpy()[cand_idx[r, b].numpy() >= 0] for r in range(R)])
            keep = np.sort(g[np.lexsort((-g, -s))[:k]])
            mine = (keep >= bases[rank]) & (keep < (bases[rank + 1] if rank + 1 < R else 1 << 30))
            out[b, :len(keep)] = np.where(mine, keep - bases[rank], -1)
        return torch.from_numpy(out.astype(np.int32))


class _NoRescale(OracleOps):
    def merge(self, shares, L, pos):
        # planted mistake: the shares' sums taken as if they shared one maximum
        sh = shares.clone()
        H = L.q.shape[1]
        sh[:, :, :H] = sh[:, :, :H].max(dim=0, keepdim=True).values.expand_as(sh[:, :, :H])
        return super().merge(sh, L, pos)


def test_planted_merge_mistakes_are_caught():
    L = make_layer("csa", seed=5, k=6, tie_pairs=[(20, 5), (33, 40), (2, 60)])
    p = torch.tensor([255, 255], dtype=torch.int32)
    with pytest.raises(AssertionError):
        _check(L, p, *_run_emulated(L, p, CP.shard_ranges(64, 2), ops=_NoRescale()))
    L["kI"][:] = L["kI"][:, :1]
    outs, idx, bases = _run_emulated(L, p, CP.shard_ranges(64, 2), ops=_TieHigh())
    assert not (_global_selection(idx, bases) == np.arange(6)[None]).all()


def test_shard_ranges():
    assert CP.shard_ranges(10, 3) == [(0, 4), (4, 3), (7, 3)]
    assert CP.shard_ranges(2, 4) == [(0, 1), (1, 1), (2, 0), (2, 0)]
    assert CP.shard_ranges(0, 1) == [(0, 0)]
    with pytest.raises(ValueError):
        CP.shard_ranges(5, 0)
    with pytest.raises(ValueError):
        CP.CPDecodeLayer(2, [0, 5], exchange=None)


# ---------------------------------------------------------------- gloo ranks

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = []
        for kind, pos in (("csa", [255, 37]), ("hca", [1023, 15])):
            L = make_layer(kind, seed=11)
            p = torch.tensor(pos, dtype=torch.int32)
            ranges = CP.shard_ranges(64, world)
            layer = CP.CPDecodeLayer(rank, [b for b, _ in ranges], CP.DistExchange(), ops=OracleOps())
            shard = shard_of(L, *ranges[rank], CP.Shard)
            out = layer(shard, p)
            ref, _ = reference(L, p)
            res.append(float(np.abs(out.numpy() - ref).max()))
        q.put((rank, res, None))
    except Exception as e:                                  # reported to the parent
        q.put((rank, None, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_match_unsharded_oracle(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, errs, exc in res:
        assert exc is None, f"rank {rank}: {exc}"
        assert max(errs) <= TOL, f"rank {rank}: max-abs {errs}"
