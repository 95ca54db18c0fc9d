"""Shared checks for the GPU parity tests.

Tolerances (stated for this path): fp32 outputs max-abs <= 1e-5; bf16 outputs
(fp32 accumulation) max-abs <= 2e-2 and relative L2 <= 5e-3; top-k index sets
exact except that indices whose oracle score lies within 1e-3 relative of the
oracle's k-th score may be swapped.
"""

import numpy as np
import torch

from oracle import csahca_oracle as O

F32_MAX_ABS = 1e-5
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
TIE_REL = 1e-3


def npy(t: torch.Tensor) -> np.ndarray:
    """Exact float64 (or int64) copy of a tensor on the host."""
    if t.dtype in (torch.int32, torch.int64, torch.uint8):
        return t.detach().cpu().numpy()
    return t.detach().cpu().to(torch.float64).numpy()


def check_close(got, ref, dtype: str, what: str = ""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - ref).max() if got.size else 0.0
    if dtype == "f32":
        assert err <= F32_MAX_ABS, f"{what}: max-abs {err:.3e} > {F32_MAX_ABS}"
    else:
        rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
        assert err <= BF16_MAX_ABS, f"{what}: max-abs {err:.3e} > {BF16_MAX_ABS}"
        assert rel <= BF16_REL_L2, f"{what}: rel-L2 {rel:.3e} > {BF16_REL_L2}"
    return err


def check_topk(got, scores, k: int, what: str = ""):
    """got: GPU index row (length k); scores: oracle scores of the visible
    entries.  Passes if the row has the right size and order, holds every
    index scoring above the tie band and none scoring below it."""
    got = np.asarray(got, np.int64)
    v = len(scores)
    if v <= k:
        want = list(range(v)) + [-1] * (k - v)
        assert list(got) == want, f"{what}: v={v} <= k={k} must select everything"
        return 0
    assert (got >= 0).all() and (got < v).all(), f"{what}: index out of range"
    assert (np.diff(got) > 0).all(), f"{what}: not sorted ascending / not unique"
    s = np.asarray(scores, np.float64)
    sk = np.sort(s)[::-1][k - 1]
    lo, hi = sk - TIE_REL * abs(sk), sk + TIE_REL * abs(sk)
    chosen = np.zeros(v, bool)
    chosen[got] = True
    missing = np.where((s > hi) & ~chosen)[0]
    extra = np.where((s < lo) & chosen)[0]
    assert missing.size == 0, f"{what}: misses {missing.size} entries above the tie band"
    assert extra.size == 0, f"{what}: holds {extra.size} entries below the tie band"
    return int(((s >= lo) & (s <= hi)).sum())


def oracle_compress(kind, inp, m, b, entries, rms_norm, gain, r):
    """Oracle entries (final rows) of sequence b for the given entry indices."""
    out = []
    for i in entries:
        if kind == "csa":
            lo = max(0, (i - 1) * m)
            sl = slice(lo, (i + 1) * m)
            pooled = O.csa_pool(npy(inp["a"][b, sl]), npy(inp["b"][b, sl]), npy(inp["za"][b, sl]),
                                npy(inp["zb"][b, sl]), npy(inp["bias_a"]), npy(inp["bias_b"]), m)
            row = pooled[-1]
        else:
            sl = slice(i * m, (i + 1) * m)
            row = O.hca_pool(npy(inp["a"][b, sl]), npy(inp["za"][b, sl]), npy(inp["bias_a"]), m)[0]
        out.append(O.finish_rows(row[None], [i * m], None if gain is None else npy(gain), r,
                                 normalize=rms_norm)[0])
    return np.stack(out)
