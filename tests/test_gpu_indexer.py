"""GPU parity of indexer_topk against the float64 oracle ("Paper Breakdown:
DeepSeek-V4", section 4, DSA on Compressed KV; "How DeepSeek-V4 architecture
and training work together", "Two compressed views of one history")."""

import numpy as np
import pytest
import torch

from long_context_compressed_overlapped_b200 import api, synth
from oracle import csahca_oracle as O
from tests.helpers import check_topk, npy

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _keys_np(kI, scale, b):
    if kI.dtype == torch.uint8:
        return O.dequant_e4m3_rows(npy(kI[b]), npy(scale[b]))
    return npy(kI[b])


def _check_rows(idx, qI, w, kI, scale, q_pos, m, k, rows, scores_gpu=None):
    bands = 0
    for (b, q) in rows:
        t = int(q_pos[b, q])
        v = min(O.n_visible(t, m), kI.shape[1]) if t >= 0 else 0
        K = _keys_np(kI, scale, b)[:v]
        s = O.indexer_scores(npy(qI[b, q]), npy(w[b, q]), K)
        bands += check_topk(npy(idx[b, q]), s, k, f"b={b} q={q} t={t}")
        if scores_gpu is not None and v:
            g = npy(scores_gpu[b, q, :v])
            scale_s = np.abs(s).max() + 1e-30
            assert np.abs(g - s).max() <= 2e-5 * scale_s, f"scores b={b} q={q}"
    return bands


def test_indexer_tiny_f32():
    """tiny_csa_f32 shapes (HI = 2, dI = 32, k = 16, m = 4) at n = 512."""
    wl = synth.WORKLOADS["tiny_csa_f32"]
    D = synth.Draw(10, DEV)
    B, n, N = 1, 512, 128
    qI = D.normal("qI", (B, n, wl.HI, wl.dI), 1 / np.sqrt(wl.dI))
    w = D.normal("w", (B, n, wl.HI), 1 / np.sqrt(wl.HI))
    kI = D.normal("kI", (B, N, wl.dI), 1 / np.sqrt(wl.dI))
    q_pos = torch.arange(n, device=DEV, dtype=torch.int32)[None]
    scores = torch.full((B, n, N), float("nan"), device=DEV)
    idx = api.indexer_topk(qI, w, kI, q_pos, wl.m, wl.k, scores_out=scores)
    _check_rows(idx, qI, w, kI, None, q_pos, wl.m, wl.k, [(0, q) for q in range(n)], scores)
    # without scores_out (workspace path) the selection is identical
    idx2 = api.indexer_topk(qI, w, kI, q_pos, wl.m, wl.k)
    assert torch.equal(idx, idx2)
    assert api.device_error() == 0


@pytest.mark.parametrize("B,n,N,k", [(2, 4096 + 5, 1024 + 1, 256), (1, 2048, 512, 1024)])
def test_indexer_bf16_prefill_shapes(B, n, N, k):
    """csa_prefill_128k head shapes (HI = 64, dI = 128) with a ragged key count
    and both v > k and v <= k queries."""
    wl = synth.WORKLOADS["csa_prefill_128k"]
    D = synth.Draw(11, DEV)
    qI = D.normal("qI", (B, n, wl.HI, wl.dI), 1.0, torch.bfloat16)
    w = D.normal("w", (B, n, wl.HI), 1 / np.sqrt(wl.HI))
    kI = D.normal("kI", (B, N, wl.dI), 1.0, torch.bfloat16)
    q_pos = torch.arange(n, device=DEV, dtype=torch.int32)[None].repeat(B, 1)
    scores = torch.zeros(B, n, N, device=DEV)
    idx = api.indexer_topk(qI, w, kI, q_pos, wl.m, k, scores_out=scores)
    rng = np.random.default_rng(0)
    qs = np.unique(np.r_[0, 2, 3, 4, 4 * k - 1, 4 * k, 4 * k + 3, n - 1, rng.integers(0, n, 40)])
    qs = qs[qs < n]
    rows = [(b, int(q)) for b in range(B) for q in qs]
    _check_rows(idx, qI, w, kI, None, q_pos, wl.m, k, rows, scores)
    assert api.device_error() == 0


@pytest.mark.parametrize("fp8", [False, True])
def test_indexer_decode_shapes(fp8):
    """One query per sequence against a long key cache (decode), bf16 keys or
    e4m3 keys with one scale per 128-element row."""
    wl = synth.WORKLOADS["decode_1m" if fp8 else "decode_256k"]
    D = synth.Draw(12, DEV)
    B, ctx = 3, 65536
    N = ctx // wl.m
    qI = D.normal("qI", (B, 1, wl.HI, wl.dI), 1.0, torch.bfloat16)
    w = D.normal("w", (B, 1, wl.HI), 1 / np.sqrt(wl.HI))
    kI = D.normal("kI", (B, N, wl.dI), 1.0, torch.bfloat16)
    scale = None
    if fp8:
        kI, scale = synth.quantize_e4m3_rows(kI)
    q_pos = torch.tensor([[ctx], [ctx - 1], [4 * 1000 + 2]], device=DEV, dtype=torch.int32)
    idx = api.indexer_topk(qI, w, kI, q_pos, wl.m, wl.k, kI_scale=scale)
    _check_rows(idx, qI, w, kI, scale, q_pos, wl.m, wl.k, [(b, 0) for b in range(B)])
    assert api.device_error() == 0


def test_indexer_decode_e4m3_long_rows():
    """e4m3 keys with rows longer than one CTA's top-k (the FP8 indexer builds
    the row histograms while scoring): a ragged key count, v > k, v = k + 1
    and v < k rows."""
    wl = synth.WORKLOADS["decode_1m"]
    D = synth.Draw(14, DEV)
    B, N = 4, 40001
    qI = D.normal("qI", (B, 1, wl.HI, wl.dI), 1.0, torch.bfloat16)
    w = D.normal("w", (B, 1, wl.HI), 1 / np.sqrt(wl.HI))
    kI, scale = synth.quantize_e4m3_rows(D.normal("kI", (B, N, wl.dI), 1.0, torch.bfloat16))
    q_pos = torch.tensor([[4 * N + 3], [4 * N - 9], [4 * (wl.k + 1) - 1], [4 * 700 + 2]], device=DEV,
                         dtype=torch.int32)
    idx = api.indexer_topk(qI, w, kI, q_pos, wl.m, wl.k, kI_scale=scale)
    _check_rows(idx, qI, w, kI, scale, q_pos, wl.m, wl.k, [(b, 0) for b in range(B)])
    # the same selection a second time (the scratch is reused)
    idx2 = api.indexer_topk(qI, w, kI, q_pos, wl.m, wl.k, kI_scale=scale)
    assert torch.equal(idx, idx2)
    assert api.device_error() == 0


def test_indexer_long_rows_ties_and_large_k():
    """Rows longer than one CTA's top-k (the multi-CTA select): every score
    equal (the lowest indices win, bf16 and e4m3 keys), eight distinct key
    rows (thousands of ties at the threshold, lowest indices first), and k
    above the sorted-selection limit (the bitmap selection)."""
    wl = synth.WORKLOADS["decode_1m"]
    D = synth.Draw(15, DEV)
    B, N = 2, 40001
    qI = D.normal("qI", (B, 1, wl.HI, wl.dI), 1.0, torch.bfloat16)
    w = D.normal("w", (B, 1, wl.HI), 1 / np.sqrt(wl.HI))
    q_pos = torch.tensor([[4 * N + 3], [4 * N - 1]], device=DEV, dtype=torch.int32)
    same = D.normal("k1", (B, 1, wl.dI), 1.0, torch.bfloat16).repeat(1, N, 1).contiguous()
    for kk, sc in ((same, None), synth.quantize_e4m3_rows(same)):
        idx = api.indexer_topk(qI, w, kk, q_pos, wl.m, 64, kI_scale=sc)
        for b in range(B):
            assert npy(idx[b, 0]).tolist() == list(range(64)), f"all-equal b={b}"
    few = D.normal("k8", (B, 8, wl.dI), 1.0, torch.bfloat16)
    kf = few[:, torch.arange(N, device=DEV) % 8].contiguous()
    idx = api.indexer_topk(qI, w, kf, q_pos, wl.m, wl.k)
    for b in range(B):
        v = min(O.n_visible(int(q_pos[b, 0]), wl.m), N)
        s = O.indexer_scores(npy(qI[b, 0]), npy(w[b, 0]), npy(kf[b])[:v])
        want = np.sort(np.argsort(-s, kind="stable")[:wl.k])
        assert npy(idx[b, 0]).tolist() == want.tolist(), f"ties b={b}"
    kr = D.normal("kr", (B, N, wl.dI), 1.0, torch.bfloat16)
    idx = api.indexer_topk(qI, w, kr, q_pos, wl.m, 5000)
    _check_rows(idx, qI, w, kr, None, q_pos, wl.m, 5000, [(b, 0) for b in range(B)])
    assert api.device_error() == 0


def test_indexer_edge_cases():
    """No visible entry (t < m - 1, negative t), exactly k visible, k = 1,
    and all-equal scores (ties go to the lower index)."""
    D = synth.Draw(13, DEV)
    HI, dI, m = 4, 64, 4
    qI = D.normal("qI", (1, 6, HI, dI), 1.0, torch.bfloat16)
    w = D.normal("w", (1, 6, HI), 0.5)
    kI = D.normal("kI", (1, 64, dI), 1.0, torch.bfloat16)
    q_pos = torch.tensor([[0, 2, -5, 4 * 8 - 1, 255, 100]], device=DEV, dtype=torch.int32)
    idx = api.indexer_topk(qI, w, kI, q_pos, m, 8)
    assert npy(idx[0, 0]).tolist() == [-1] * 8
    assert npy(idx[0, 1]).tolist() == [-1] * 8
    assert npy(idx[0, 2]).tolist() == [-1] * 8
    assert npy(idx[0, 3]).tolist() == list(range(8))            # exactly k visible
    _check_rows(idx, qI, w, kI, None, q_pos, m, 8, [(0, 4), (0, 5)])
    idx1 = api.indexer_topk(qI, w, kI, q_pos, m, 1)
    _check_rows(idx1, qI, w, kI, None, q_pos, m, 1, [(0, q) for q in range(6)])
    # identical keys: every score ties, the lowest indices win
    kc = kI[:, :1].repeat(1, 64, 1).contiguous()
    idx_t = api.indexer_topk(qI, w, kc, q_pos, m, 8)
    assert npy(idx_t[0, 4]).tolist() == list(range(8))
    assert api.device_error() == 0
