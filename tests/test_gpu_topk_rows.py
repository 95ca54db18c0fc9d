"""GPU top-k of rows up to 32,768 visible entries (the one-CTA-per-row
selection of prefill), against the oracle's selection rule applied to the
GPU's own fp32 scores: with identical scores the selection must match
exactly, ties going to the lower index ("Paper Breakdown: DeepSeek-V4",
section 4, DSA on Compressed KV: the top-k entries by I_{t,s}).

The rows cover every path of the selection: rows short enough to keep every
key, rows whose bound comes from a sample of their segments, rows where the
sample misleads (too few keys kept, or too many for the lists) and the
three-pass fallback runs, massive ties and all-equal rows."""

import numpy as np
import pytest
import torch

from long_context_compressed_overlapped_b200 import api, synth
from oracle import csahca_oracle as O
from tests.helpers import npy

pytestmark = pytest.mark.gpu
DEV = "cuda"
HI, DI, M, K = 64, 128, 4, 1024


def _positions(vs):
    """Query positions whose visible count is v (t = 4 v - 1 with m = 4)."""
    return torch.tensor([[M * v - 1 for v in vs]], device=DEV, dtype=torch.int32)


def _run_exact(kI, qI, w, pos):
    N = kI.shape[1]
    nq = pos.shape[1]
    scores = torch.zeros(1, nq, N, device=DEV)
    idx = api.indexer_topk(qI, w, kI, pos, M, K, scores_out=scores)
    for q in range(nq):
        v = min(O.n_visible(int(pos[0, q]), M), N)
        want = O.top_k_select(npy(scores[0, q, :v]), K)
        assert npy(idx[0, q]).tolist() == want.tolist(), f"query {q} (v={v})"
    assert api.device_error() == 0
    return idx


VS = [5, 1023, 1024, 1025, 3000, 4095, 4096, 4097, 6001, 8192, 12345, 20000, 32767, 32768]


def test_rows_gaussian_all_lengths():
    """Gaussian keys, queries and weights; one query per visible length."""
    N = 32768
    D = synth.Draw(31, DEV)
    kI = D.normal("kI", (1, N, DI), 1.0, torch.bfloat16)
    qI = D.normal("qI", (1, len(VS), HI, DI), 1.0, torch.bfloat16)
    w = D.normal("w", (1, len(VS), HI), 1 / 8)
    _run_exact(kI, qI, w, _positions(VS))


def _one_dim_keys(vals):
    """Keys whose score is a monotone function of vals (query and weight on
    dimension 0 only, both positive)."""
    N = vals.shape[0]
    kI = torch.zeros(1, N, DI, device=DEV)
    kI[0, :, 0] = vals
    return kI.to(torch.bfloat16)


def _one_dim_query(nq):
    qI = torch.zeros(1, nq, HI, DI, device=DEV)
    qI[..., 0, 0] = 1.0
    w = torch.zeros(1, nq, HI, device=DEV)
    w[..., 0] = 1.0
    return qI.to(torch.bfloat16), w


def test_rows_sample_misleads():
    """Keys in the sampled segments (one 32-key segment in 8) larger than the
    rest, and the reverse: the sample's bound keeps too few keys, or too many
    for the lists, and the three passes decide."""
    N = 32768
    j = torch.arange(N, device=DEV)
    sampled = ((j // 32) % 8) == 0
    D = synth.Draw(32, DEV)
    noise = D.normal("n", (N,), 1.0).abs() * 0.01
    vs = [4097, 9000, 20000, 32768]
    qI, w = _one_dim_query(len(vs))
    for hi_in_sample in (True, False):
        vals = torch.where(sampled == hi_in_sample, 4.0 + noise, 1.0 + noise)
        _run_exact(_one_dim_keys(vals), qI, w, _positions(vs))


def test_rows_massive_ties_and_all_equal():
    """Six key levels (thousands of equal scores at the threshold) and one
    level (every score equal: the k lowest indices)."""
    N = 32768
    D = synth.Draw(33, DEV)
    lev = D.integers("lev", 0, 6, (N,)).float() * 0.25 + 0.5
    vs = [1025, 4097, 16000, 32768]
    qI, w = _one_dim_query(len(vs))
    _run_exact(_one_dim_keys(lev), qI, w, _positions(vs))
    idx = _run_exact(_one_dim_keys(torch.full((N,), 0.75, device=DEV)), qI, w, _positions(vs))
    for q in range(len(vs)):
        assert npy(idx[0, q]).tolist() == list(range(K))
