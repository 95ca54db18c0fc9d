"""GPU top-k over long rows (the multi-CTA path used when a row can hold more
than 32,768 visible entries, as in decode at long context), against the
oracle's selection rule applied to the GPU's own fp32 scores: with identical
scores on both sides the selection must match exactly, including ties, which
go to the lower index ("Paper Breakdown: DeepSeek-V4", section 4, DSA on
Compressed KV: the top-k entries by I_{t,s})."""

import pytest
import torch

from long_context_compressed_overlapped_b200 import api, synth
from oracle import csahca_oracle as O
from tests.helpers import check_topk, npy

pytestmark = pytest.mark.gpu
DEV = "cuda"
HI, DI, M, K = 64, 128, 4, 1024


def _run(kI, qI, w, pos):
    B, N, _ = kI.shape
    scores = torch.zeros(B, 1, N, device=DEV)
    idx = api.indexer_topk(qI, w, kI, pos, M, K, scores_out=scores)
    return idx, scores


def _exact(idx, scores, pos, N):
    for b in range(idx.shape[0]):
        v = min(O.n_visible(int(pos[b, 0]), M), N)
        want = O.top_k_select(npy(scores[b, 0, :v]), K)
        assert npy(idx[b, 0]).tolist() == want.tolist(), f"row {b} (v={v})"


def test_topk_long_rows_with_massive_ties():
    """Key values from 6 levels make thousands of exactly equal scores in the
    threshold bin; rows of different visible lengths (v > k, v = k + 1, v = k,
    v < k)."""
    N = 50000 + 17
    D = synth.Draw(21, DEV)
    lev = D.integers("lev", 0, 6, (4, N, 1)).float() * 0.25 + 0.5
    kI = torch.zeros(4, N, DI, device=DEV)
    kI[..., :1] = lev
    kI = kI.to(torch.bfloat16)
    qI = torch.zeros(4, 1, HI, DI, device=DEV)
    qI[..., 0, 0] = 1.0
    qI = qI.to(torch.bfloat16)
    w = torch.zeros(4, 1, HI, device=DEV)
    w[..., 0] = 1.0
    pos = torch.tensor([[4 * N + 3], [4 * (K + 1) - 1], [4 * K - 1], [4 * 100]], device=DEV,
                       dtype=torch.int32)
    idx, scores = _run(kI, qI, w, pos)
    _exact(idx, scores, pos, N)
    assert api.device_error() == 0


def test_topk_long_rows_gaussian_and_negative():
    """Gaussian keys and weights (continuous scores) and a row whose weights
    are all negative (every score <= 0), checked exactly on the GPU's scores
    and against the float64 oracle scores with the 1e-3 tie band."""
    N = 70000
    D = synth.Draw(22, DEV)
    kI = D.normal("kI", (3, N, DI), 1.0, torch.bfloat16)
    qI = D.normal("qI", (3, 1, HI, DI), 1.0, torch.bfloat16)
    w = D.normal("w", (3, 1, HI), 1 / 8)
    w[2] = -w[2].abs()
    pos = torch.tensor([[4 * N - 1], [4 * 50000 + 2], [4 * N + 100]], device=DEV, dtype=torch.int32)
    idx, scores = _run(kI, qI, w, pos)
    _exact(idx, scores, pos, N)
    for b in range(3):
        v = min(O.n_visible(int(pos[b, 0]), M), N)
        s = O.indexer_scores(npy(qI[b, 0]), npy(w[b, 0]), npy(kI[b, :v]))
        check_topk(npy(idx[b, 0]), s, K, f"row {b}")
    assert api.device_error() == 0


def test_topk_long_rows_all_equal():
    """Every key identical: all scores tie and the k lowest indices win."""
    N = 40000
    kI = torch.full((2, N, DI), 0.5, device=DEV).to(torch.bfloat16)
    D = synth.Draw(23, DEV)
    qI = D.normal("qI", (2, 1, HI, DI), 1.0, torch.bfloat16)
    w = torch.full((2, 1, HI), 0.125, device=DEV)
    pos = torch.tensor([[4 * N - 1], [4 * 30000]], device=DEV, dtype=torch.int32)
    idx, scores = _run(kI, qI, w, pos)
    assert npy(idx[0, 0]).tolist() == list(range(K))
    assert npy(idx[1, 0]).tolist() == list(range(K))
    assert api.device_error() == 0


def test_topk_repeated_calls_are_identical():
    """The scratch is re-initialised on every call: two calls in a row give
    the same selection."""
    N = 65536
    D = synth.Draw(24, DEV)
    kI = D.normal("kI", (2, N, DI), 1.0, torch.bfloat16)
    qI = D.normal("qI", (2, 1, HI, DI), 1.0, torch.bfloat16)
    w = D.normal("w", (2, 1, HI), 1 / 8)
    pos = torch.tensor([[4 * N - 1], [4 * N - 1]], device=DEV, dtype=torch.int32)
    a = api.indexer_topk(qI, w, kI, pos, M, K)
    b = api.indexer_topk(qI, w, kI, pos, M, K)
    assert torch.equal(a, b)
    assert api.device_error() == 0
