"""The four compute steps of a context-parallel decode layer written out in
float64 from the oracle's definitions (test infrastructure: these stand in
for the library's kernels when the schedule runs on CPU ranks).

The merge rules follow from the definitions alone: the top-k of a union is
the top-k of the union of the parts' top-k lists (ties to the lower global
entry); and a softmax over a union of key sets with the sink is the parts'
partial sums rescaled to a common maximum ("Paper Breakdown: DeepSeek-V4",
section 4, DSA on compressed KV and the attention sink)."""

import numpy as np
import torch

from oracle import csahca_oracle as O

LOG2E = 1.0 / np.log(2.0)


def _np(t):
    return None if t is None else t.detach().cpu().to(torch.float64).numpy()


def local_visible(t: int, m: int, base: int, n: int) -> int:
    return int(min(max(O.n_visible(t, m) - base, 0), n)) if t >= 0 else 0


class OracleOps:
    """Per-rank steps on host tensors, float64."""

    def local_topk(self, L, pos, k):
        B = L.q.shape[0]
        idx = np.full((B, k), -1, np.int64)
        sc = np.full((B, k), -np.inf)
        for b in range(B):
            t = int(pos[b])
            v = local_visible(t, L.m, L.entry_base, L.kI.shape[1])
            s = O.indexer_scores(_np(L.qI[b]), _np(L.wI[b]), _np(L.kI[b])[:v])
            sel = O.top_k_select(s, k)
            idx[b] = sel
            sc[b, sel >= 0] = s[sel[sel >= 0]]
        return torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(sc)

    def topk_merge(self, cand_idx, cand_scores, bases, rank):
        R, B, k = cand_idx.shape
        out = np.full((B, k), -1, np.int64)
        ci, cs = cand_idx.numpy().astype(np.int64), cand_scores.numpy()
        for b in range(B):
            g, s, owner = [], [], []
            for r in range(R):
                ok = ci[r, b] >= 0
                g += list(bases[r] + ci[r, b][ok])
                s += list(cs[r, b][ok])
                owner += [r] * int(ok.sum())
            g, s, owner = np.array(g, np.int64), np.array(s), np.array(owner)
            if len(g) == 0:
                continue
            order = np.lexsort((g, -s))[:k]              # score desc, then lower entry
            keep = order[np.argsort(g[order])]            # ascending global entry
            loc = np.where(owner[keep] == rank, g[keep] - bases[rank], -1)
            out[b, :len(keep)] = loc
        return torch.from_numpy(out.astype(np.int32))

    def local_share(self, L, pos, idx_local, skip_window):
        B, H, d = L.q.shape
        tau = 1.0 / np.sqrt(d)
        w = L.win.shape[1]
        kv = _np(L.kv)
        out = np.zeros((B, 2 * H + H * d))
        for b in range(B):
            t = int(pos[b])
            qt = O.finish_rows(_np(L.q[b]), t, _np(L.q_gain), L.rope_dims)
            if L.kind == "csa":
                sel = idx_local[b].numpy().astype(np.int64)
                keys = kv[b][sel[sel >= 0]]
            else:
                keys = kv[b][:local_visible(t, L.m, L.entry_base, kv.shape[1])]
            if not skip_window and w > 0:
                keys = np.concatenate([keys, _np(L.win[b])[O.window_positions(t, w) % w]], axis=0)
            mx = np.full(H, -np.inf)
            lsum = np.zeros(H)
            o = np.zeros((H, d))
            if keys.shape[0]:
                s2 = tau * (qt @ keys.T) * LOG2E              # logits in base-2 units
                mx = s2.max(axis=1)
                e = np.exp2(s2 - mx[:, None])
                lsum = e.sum(axis=1)
                o = (e @ keys) / lsum[:, None]
            out[b, :H], out[b, H:2 * H], out[b, 2 * H:] = mx, lsum, o.reshape(-1)
        return torch.from_numpy(out)

    def merge(self, shares, L, pos):
        R, B, _ = shares.shape
        H, d = L.q.shape[1:]
        sh = shares.numpy()
        z2 = _np(L.sinks) * LOG2E
        out = np.zeros((B, H, d))
        for b in range(B):
            mx, lsum = sh[:, b, :H], sh[:, b, H:2 * H]
            o = sh[:, b, 2 * H:].reshape(R, H, d)
            M = np.maximum(z2, mx.max(axis=0))
            c = np.where(np.isneginf(mx), 0.0, lsum * np.exp2(mx - M[None]))
            den = c.sum(axis=0) + np.exp2(z2 - M)
            y = np.einsum("rh,rhd->hd", c, o) / den[:, None]
            out[b] = O.rope(y, -int(pos[b]), L.rope_dims)
        return torch.from_numpy(out)


def make_layer(kind: str, seed: int, *, B=2, H=4, d=64, r=16, m=4, HI=2, dI=32, k=8, w=16, n_entries=64,
               tie_pairs=()):
    """A small decode layer over a whole cache (float64 host tensors): q,
    final cache rows, window ring, sinks, gain; CSA also indexer query,
    weights and keys.  tie_pairs: (i, j) entries whose indexer keys are made
    equal (scores tie)."""
    g = np.random.default_rng(seed)
    L = dict(kind=kind, m=m if kind == "csa" else 16, rope_dims=r, k=k if kind == "csa" else 0,
             q=g.standard_normal((B, H, d)), kv=g.standard_normal((B, n_entries, d)) / np.sqrt(d) * 4,
             win=g.standard_normal((B, w, d)) / np.sqrt(d) * 4, sinks=g.standard_normal(H),
             q_gain=1.0 + 0.1 * g.standard_normal(d))
    if kind == "csa":
        kI = g.standard_normal((B, n_entries, dI)) / np.sqrt(dI)
        for i, j in tie_pairs:
            kI[:, j] = kI[:, i]
        L.update(qI=g.standard_normal((B, HI, dI)), wI=np.abs(g.standard_normal((B, HI))), kI=kI)
    return {key: (torch.from_numpy(v) if isinstance(v, np.ndarray) else v) for key, v in L.items()}


def shard_of(L: dict, base: int, n: int, shard_cls):
    """The Shard of entries base .. base + n - 1 of a whole-cache layer."""
    kw = dict(kind=L["kind"], entry_base=base, q=L["q"], kv=L["kv"][:, base:base + n].contiguous(), win=L["win"],
              sinks=L["sinks"], m=L["m"], rope_dims=L["rope_dims"], q_gain=L["q_gain"], k=L["k"])
    if L["kind"] == "csa":
        kw.update(qI=L["qI"], wI=L["wI"], kI=L["kI"][:, base:base + n].contiguous())
    return shard_cls(**kw)


def reference(L: dict, pos):
    """The unsharded layer: the oracle's top-k over the whole cache and
    decode_attention (window and sink included); returns (out [B, H, d],
    sel [B, k] or None)."""
    B, H, d = L["q"].shape
    w = L["win"].shape[1]
    outs, sels = [], []
    for b in range(B):
        t = int(pos[b])
        sel = None
        if L["kind"] == "csa":
            v = min(O.n_visible(t, L["m"]), L["kI"].shape[1])
            s = O.indexer_scores(_np(L["qI"][b]), _np(L["wI"][b]), _np(L["kI"][b])[:v])
            sel = O.top_k_select(s, L["k"])
            sels.append(sel)
        outs.append(O.decode_attention(L["kind"], _np(L["q"][b]), t, _np(L["kv"][b]), _np(L["win"][b]),
                                       _np(L["sinks"]), m=L["m"], w=w, r=L["rope_dims"], q_gain=_np(L["q_gain"]),
                                       sel=sel))
    return np.stack(outs), (np.stack(sels) if sels else None)
