"""GPU parity of the context-parallel path ("Paper Breakdown: DeepSeek-V4",
infrastructure table, "2-Stage Context Parallel"): the ranks of a layer run
on one GPU, one after another, in the schedule of
context_parallel.CPDecodeLayer (each rank's shard of the cache, the
exchanges done by stacking the ranks' buffers; no kernel waits on another).
The global selection must pass the top-k rule against the oracle over the
whole cache and equal the one-GPU selection, and the output must match the
oracle (bf16 tolerances) and the one-GPU output.  The merge kernels are also
checked alone against float64 restatements, and decode_compress with
entry_base against the unsharded call."""

import ctypes as C

import numpy as np
import pytest
import torch

from long_context_compressed_overlapped_b200 import api, context_parallel as CP, native, runtime, synth
from oracle import csahca_oracle as O
from tests.helpers import check_close, check_topk, npy

pytestmark = pytest.mark.gpu
DEV = "cuda"
LOG2E = 1.0 / np.log(2.0)


def _shards(L, wl, ranges):
    out = []
    for base, n in ranges:
        kw = dict(kind=L["kind"], entry_base=base, q=L["q"], kv=L["kv"][:, base:base + n].contiguous(),
                  win=L["win"], sinks=L["sinks"], m=L["m"], rope_dims=wl.r, q_gain=L["q_gain"])
        if L["kind"] == "csa":
            kw.update(qI=L["qI"], wI=L["w"], kI=L["kI"][:, base:base + n].contiguous(),
                      kI_scale=None if L["kI_scale"] is None else L["kI_scale"][:, base:base + n].contiguous(),
                      k=wl.k)
        out.append(CP.Shard(**kw))
    return out


def _run_ranks(L, wl, ranges, pos):
    bases = [b for b, _ in ranges]
    ranks = [CP.CPDecodeLayer(r, bases, exchange=None) for r in range(len(ranges))]
    shards = _shards(L, wl, ranges)
    idx = [None] * len(ranges)
    if L["kind"] == "csa":
        cands = [cp.local_candidates(s, pos) for cp, s in zip(ranks, shards)]
        ci = torch.stack([c[0] for c in cands])
        cs = torch.stack([c[1] for c in cands])
        idx = [cp.merge_candidates(ci, cs) for cp in ranks]
        g, _ = api.cp_topk_merge(ci, cs, bases, 0)
    else:
        g = None
    shares = torch.stack([cp.local_share(s, pos, ix) for cp, s, ix in zip(ranks, shards, idx)])
    outs = [cp.merge_shares(shares, s, pos) for cp, s in zip(ranks, shards)]
    return outs, idx, g


def _global_from_local(idx, bases):
    B, k = idx[0].shape
    rows = []
    for b in range(B):
        gl = sorted(int(bases[r] + x) for r, ix in enumerate(idx) for x in npy(ix[b]).tolist() if x >= 0)
        rows.append(gl + [-1] * (k - len(gl)))
    return np.array(rows)


@pytest.mark.parametrize("wl_name,R", [("decode_1m", 2), ("decode_1m", 3), ("decode_256k", 2),
                                       ("decode_1m_fp8kv", 3)])
def test_context_parallel_layers(wl_name, R):
    """CSA and HCA layers of decode_1m shapes (e4m3 indexer keys), of
    decode_256k (bf16 keys) and with FP8 KV rows, split over R ranks; one
    sequence sees every shard, one only the first."""
    wl = synth.WORKLOADS[wl_name]
    ctx = 32768 + 130
    layers = synth.decode_inputs(wl, DEV, ctx=ctx, B=2, layers=("csa", "hca"))
    for L in layers:
        N = L["kv"].shape[1]
        ranges = CP.shard_ranges(N, R)
        early = (ranges[0][1] - 10) * L["m"] + 3              # visible entries end inside shard 0
        pos = torch.tensor([ctx, early], dtype=torch.int32, device=DEV)
        L["pos"] = pos
        outs, idx, g = _run_ranks(L, wl, ranges, pos)
        # the one-GPU layer
        idx1 = torch.empty(2, wl.k, dtype=torch.int32, device=DEV) if L["kind"] == "csa" else None
        kw = dict(m=L["m"], rope_dims=wl.r, q_gain=L["q_gain"])
        if L["kind"] == "csa":
            kw.update(k=wl.k, qI=L["qI"], wI=L["w"], kI=L["kI"], kI_scale=L["kI_scale"], idx_out=idx1)
        out1 = api.compressed_attn_decode(L["kind"], L["q"], pos, L["kv"], L["win"], L["sinks"], **kw)
        bases = [b for b, _ in ranges]
        kv_rows = [(synth.unpack_kv_rows_fp8(L["kv"][b], wl.d, wl.r) if wl.fp8_kv else None) for b in range(2)]
        for b in range(2):
            t = int(pos[b])
            sel = None
            if L["kind"] == "csa":
                gsel = _global_from_local(idx, bases)[b]
                assert (npy(g[b]) == gsel).all(), "idx_global differs from the union of the local rows"
                assert (gsel == npy(idx1[b])).all(), "context-parallel selection differs from one GPU's"
                v = min(O.n_visible(t, L["m"]), N)
                K = (O.dequant_e4m3_rows(npy(L["kI"][b, :v]), npy(L["kI_scale"][b, :v]))
                     if L["kI_scale"] is not None else npy(L["kI"][b, :v]))
                check_topk(gsel, O.indexer_scores(npy(L["qI"][b]), npy(L["w"][b]), K), wl.k, f"cp b={b}")
                sel = gsel
            rows = (O.dequant_kv_rows_fp8(*(npy(x) for x in kv_rows[b])) if wl.fp8_kv else npy(L["kv"][b]))
            ref = O.decode_attention(L["kind"], npy(L["q"][b]), t, rows, npy(L["win"][b]), npy(L["sinks"]),
                                     m=L["m"], w=wl.w, r=wl.r, q_gain=npy(L["q_gain"]), sel=sel)
            for r, o in enumerate(outs):
                check_close(npy(o[b]), ref, "bf16", f"{wl_name} {L['kind']} R={R} rank {r} b={b}")
            check_close(npy(outs[0][b]), npy(out1[b]), "bf16", f"{L['kind']} cp vs one GPU b={b}")
    assert api.device_error() == 0


def test_cp_topk_merge_kernel():
    """cp_topk_merge alone on random candidates with exact ties across ranks,
    padded lists, R = 1 .. 8 and k up to 2048, against a float64
    restatement of the rule (score descending, then lower global entry)."""
    g = np.random.default_rng(0)
    for R, k, rows in ((1, 16, 3), (2, 1024, 4), (3, 100, 2), (8, 2048, 2), (5, 7, 5)):
        # disjoint shards: local rows below 3k, shards at least 3k long
        bases = np.cumsum([0] + list(g.integers(3 * k, 5 * k, R - 1))).tolist()
        ci = np.full((R, rows, k), -1, np.int32)
        cs = np.full((R, rows, k), -np.inf, np.float32)
        for r in range(R):
            for row in range(rows):
                n = int(g.integers(0, k + 1)) if r % 2 else k
                loc = np.sort(g.choice(3 * k, n, replace=False)).astype(np.int32)
                ci[r, row, :n] = loc
                cs[r, row, :n] = np.round(g.standard_normal(n) * 4) / 4      # many exact ties
        want = np.full((rows, k), -1, np.int64)
        for row in range(rows):
            gl = np.concatenate([bases[r] + ci[r, row][ci[r, row] >= 0] for r in range(R)]).astype(np.int64)
            sc = np.concatenate([cs[r, row][ci[r, row] >= 0] for r in range(R)]).astype(np.float64)
            keep = np.sort(gl[np.lexsort((gl, -sc))[:k]])
            want[row, :len(keep)] = keep
        cit, cst = torch.from_numpy(ci).to(DEV), torch.from_numpy(cs).to(DEV)
        for rank in range(R):
            gout, lout = api.cp_topk_merge(cit, cst, bases, rank)
            assert (npy(gout) == want).all(), f"R={R} k={k}"
            lo = bases[rank]
            hi = bases[rank + 1] if rank + 1 < R else 1 << 30
            mine = (want >= lo) & (want < hi)
            assert (npy(lout) == np.where(mine, want - lo, -1)).all(), f"R={R} rank={rank} local rows"
    assert api.device_error() == 0


def test_cp_attn_merge_kernel():
    """cp_attn_merge alone: random shares (some ranks empty: mx = -inf,
    l = 0), sinks, positions with RoPE de-rotation, bf16 and fp32 outputs,
    against a float64 restatement."""
    g = np.random.default_rng(1)
    R, rows, H, d, r = 3, 4, 64, 512, 64
    mx = g.standard_normal((R, rows, H)) * 3
    mx[1, 2] = -np.inf
    lsum = np.abs(g.standard_normal((R, rows, H))) * 10 + 1
    lsum[1, 2] = 0
    o = g.standard_normal((R, rows, H, d))
    o[1, 2] = 0
    sh = np.concatenate([mx, lsum, o.reshape(R, rows, H * d)], axis=2).astype(np.float32)
    sinks = g.standard_normal(H).astype(np.float32)
    pos = np.array([0, 5, 1048576, 77], np.int32)
    shf = sh.astype(np.float64)
    want = np.zeros((rows, H, d))
    for row in range(rows):
        z2 = sinks.astype(np.float64) * LOG2E
        m_ = shf[:, row, :H]
        M = np.maximum(z2, m_.max(axis=0))
        c = np.where(np.isneginf(m_), 0.0, shf[:, row, H:2 * H] * np.exp2(m_ - M[None]))
        den = c.sum(axis=0) + np.exp2(z2 - M)
        y = np.einsum("rh,rhd->hd", c, shf[:, row, 2 * H:].reshape(R, H, d)) / den[:, None]
        want[row] = O.rope(y, -int(pos[row]), r)
    for dt, kind in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
        out = api.cp_attn_merge(torch.from_numpy(sh).to(DEV), torch.from_numpy(sinks).to(DEV),
                                torch.from_numpy(pos).to(DEV), H=H, d=d, rope_dims=r, dtype=dt)
        tol = 1e-4 if kind == "f32" else None
        if tol:
            err = np.abs(npy(out) - want).max()
            assert err <= tol, f"fp32 merge max-abs {err:.3e}"
        else:
            check_close(npy(out), want, "bf16", "bf16 merge")
    assert api.device_error() == 0


def test_decode_compress_into_a_shard():
    """decode_compress with entry_base: the completed entry lands in local
    row i - entry_base of the shard that holds it, byte for byte as the
    unsharded call writes row i (cache row and e4m3 indexer key), and a
    shard that does not hold entry i is left untouched."""
    wl = synth.WORKLOADS["decode_1m"]
    ctx = (1 << 15) - 1                                   # completes CSA entry 8191 and HCA entry 255
    for L in synth.decode_inputs(wl, DEV, ctx=ctx, B=2, layers=("csa", "hca")):
        m = L["m"]
        i = (ctx + 1) // m - 1
        N = L["kv"].shape[1]
        full = {n: L[n].clone() for n in ("kv", "ring", "win") + (("kI", "kI_scale", "iring") if L["kind"] == "csa"
                                                                  else ())}
        api_args, keep = runtime.compress_args(wl, {**L, **{n: full[n] for n in full}})
        native.check(native.lib().decode_compress(C.byref(api_args), torch.cuda.current_stream().cuda_stream),
                     "decode_compress")
        for base, n in ((N - 64, 64), (0, N - 64)):
            part = {nm: L[nm].clone() for nm in full}
            sh = dict(L)
            sh.update(part)
            sh["kv"] = part["kv"][:, base:base + n].contiguous()
            if L["kind"] == "csa":
                sh["kI"] = part["kI"][:, base:base + n].contiguous()
                sh["kI_scale"] = part["kI_scale"][:, base:base + n].contiguous()
            before = sh["kv"].clone()
            a2, keep2 = runtime.compress_args(wl, sh, entry_base=base)
            native.check(native.lib().decode_compress(C.byref(a2), torch.cuda.current_stream().cuda_stream),
                         "decode_compress (shard)")
            torch.cuda.synchronize()
            if base <= i < base + n:
                assert torch.equal(sh["kv"][:, i - base], full["kv"][:, i]), L["kind"]
                if L["kind"] == "csa":
                    assert torch.equal(sh["kI"][:, i - base], full["kI"][:, i])
                    assert torch.equal(sh["kI_scale"][:, i - base], full["kI_scale"][:, i])
            else:
                assert torch.equal(sh["kv"], before), f"{L['kind']}: a shard without entry {i} was written"
            assert torch.equal(sh["win"], full["win"]) and torch.equal(sh["ring"], full["ring"])
    assert api.device_error() == 0
