"""GPU parity of compressed_attn_prefill against the float64 oracle
("Paper Breakdown: DeepSeek-V4", section 4: MQA core attention, sliding
window, HCA dense attention, attention sink, RMSNorm, partial RoPE; "Inside
DeepSeek V4", "Local window")."""

import numpy as np
import pytest
import torch

from long_context_compressed_overlapped_b200 import api, synth
from oracle import csahca_oracle as O
from tests.helpers import check_close, npy

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _sample(n, extra, seed=0, count=24):
    rng = np.random.default_rng(seed)
    s = np.unique(np.r_[extra, rng.integers(0, n, count)])
    return s[(s >= 0) & (s < n)]


def _prefill_layer(wl, n, B):
    """Compressed rows (GPU compressor; both sides then read the same rows),
    raw window rows and queries."""
    inp = synth.prefill_inputs(wl, DEV, n=n, B=B)
    kvi = inp["kv"]
    m = wl.m if wl.kind == "csa" else wl.m_hca
    if wl.kind == "csa":
        kv = api.csa_compress(kvi["a"], kvi["b"], kvi["za"], kvi["zb"], kvi["bias_a"],
                              kvi["bias_b"], m, gain=inp["kv_gain"], rope_dims=wl.r)
    else:
        kv = api.hca_compress(kvi["a"], kvi["za"], kvi["bias_a"], m, gain=inp["kv_gain"],
                              rope_dims=wl.r)
    return inp, kv, m


def _oracle_rows(kind, inp, kv, idx, wl, m, b, rows):
    rows = np.asarray(rows)
    sel = torch.as_tensor(rows, device=inp["q"].device)
    return O.prefill_attention(kind, npy(inp["q"][b].index_select(0, sel)), npy(kv[b]),
                               npy(inp["kv_win"][b]), npy(inp["sinks"]), m=m, w=wl.w, r=wl.r,
                               q_gain=npy(inp["q_gain"]), kv_gain=npy(inp["kv_gain"]),
                               idx=None if idx is None else npy(idx[b]), rows=rows,
                               q_holds_rows=True)


def test_prefill_csa_tiny_f32():
    """tiny_csa_f32 end to end on the GPU (compress -> indexer -> attention);
    output parity uses the GPU's own index set on the oracle side."""
    wl = synth.WORKLOADS["tiny_csa_f32"]
    inp, kv, m = _prefill_layer(wl, wl.n, wl.B)
    ik = inp["ik"]
    kI = api.csa_compress(ik["a"], ik["b"], ik["za"], ik["zb"], ik["bias_a"], ik["bias_b"], m,
                          rms_norm=False)
    q_pos = torch.arange(wl.n, device=DEV, dtype=torch.int32)[None]
    idx = api.indexer_topk(inp["qI"], inp["w"], kI, q_pos, m, wl.k)
    out = api.compressed_attn_prefill("csa", inp["q"], kv, inp["kv_win"], inp["sinks"], m=m,
                                      w=wl.w, rope_dims=wl.r, idx=idx, q_gain=inp["q_gain"],
                                      kv_gain=inp["kv_gain"])
    ref = _oracle_rows("csa", inp, kv, idx, wl, m, 0, np.arange(wl.n))
    check_close(npy(out[0]), ref, "f32", "tiny csa prefill")
    assert api.device_error() == 0


def test_prefill_hca_8k_bf16_full_size():
    """hca_8k_bf16 at full size (B = 2, n = 8192, H = 16, d = 128, m' = 128,
    w = 128) on sampled queries, including t < m', t < w and t = n - 1."""
    wl = synth.WORKLOADS["hca_8k_bf16"]
    inp, kv, m = _prefill_layer(wl, wl.n, wl.B)
    out = api.compressed_attn_prefill("hca", inp["q"], kv, inp["kv_win"], inp["sinks"], m=m,
                                      w=wl.w, rope_dims=wl.r, q_gain=inp["q_gain"],
                                      kv_gain=inp["kv_gain"])
    for b in range(wl.B):
        rows = _sample(wl.n, [0, 1, 126, 127, 128, 255, 256, wl.n - 1], seed=b)
        ref = _oracle_rows("hca", inp, kv, None, wl, m, b, rows)
        check_close(npy(out[b, rows]), ref, "bf16", f"hca b={b}")
    assert api.device_error() == 0


def test_prefill_csa_bf16_prefill_shapes():
    """csa_prefill_128k head shapes (H = 64, d = 512, r = 64, k = 1024,
    w = 128) at n = 4096 + 3, with the GPU's selection."""
    wl = synth.WORKLOADS["csa_prefill_128k"]
    n = 4096 + 3
    inp, kv, m = _prefill_layer(wl, n, 1)
    ik = inp["ik"]
    kI = api.csa_compress(ik["a"], ik["b"], ik["za"], ik["zb"], ik["bias_a"], ik["bias_b"], m,
                          rms_norm=False)
    q_pos = torch.arange(n, device=DEV, dtype=torch.int32)[None]
    idx = api.indexer_topk(inp["qI"], inp["w"], kI, q_pos, m, wl.k)
    out = api.compressed_attn_prefill("csa", inp["q"], kv, inp["kv_win"], inp["sinks"], m=m,
                                      w=wl.w, rope_dims=wl.r, idx=idx, q_gain=inp["q_gain"],
                                      kv_gain=inp["kv_gain"])
    rows = _sample(n, [0, 3, 4, 127, 128, 4095, 4096, n - 1], count=12)
    ref = _oracle_rows("csa", inp, kv, idx, wl, m, 0, rows)
    check_close(npy(out[0, rows]), ref, "bf16", "csa prefill")
    assert api.device_error() == 0


def test_prefill_csa_tc_ragged_tiles():
    """Tensor-core CSA prefill (H = 64, d = 512) with k and w that are not
    multiples of the key tile (k = 200: a full tile of selected rows and a
    ragged one; w = 100: one ragged window tile), two sequences, and queries
    with fewer visible entries than k (lists padded with -1) or a window
    clipped at t = 0."""
    base = synth.WORKLOADS["csa_prefill_128k"]
    wl = synth.Workload(**{**base.__dict__, "k": 200, "w": 100})
    n, B = 1500 + 7, 2
    inp, kv, m = _prefill_layer(wl, n, B)
    ik = inp["ik"]
    kI = api.csa_compress(ik["a"], ik["b"], ik["za"], ik["zb"], ik["bias_a"], ik["bias_b"], m,
                          rms_norm=False)
    q_pos = torch.arange(n, device=DEV, dtype=torch.int32)[None].expand(B, n).contiguous()
    idx = api.indexer_topk(inp["qI"], inp["w"], kI, q_pos, m, wl.k)
    out = api.compressed_attn_prefill("csa", inp["q"], kv, inp["kv_win"], inp["sinks"], m=m,
                                      w=wl.w, rope_dims=wl.r, idx=idx, q_gain=inp["q_gain"],
                                      kv_gain=inp["kv_gain"])
    for b in range(B):
        rows = _sample(n, [0, 1, 3, 63, 64, 99, 100, 255, 256, 4 * wl.k - 1, 4 * wl.k, n - 1], seed=7 + b,
                       count=10)
        ref = _oracle_rows("csa", inp, kv, idx, wl, m, b, rows)
        check_close(npy(out[b, rows]), ref, "bf16", f"csa prefill ragged b={b}")
    assert api.device_error() == 0


def test_prefill_no_window_no_sink_edge():
    """w = 0 with the first queries (no visible entry): the output is 0 for
    t < m - 1 (only the sink in the denominator)."""
    wl = synth.WORKLOADS["hca_8k_bf16"]
    inp, kv, m = _prefill_layer(wl, 512, 1)
    out = api.compressed_attn_prefill("hca", inp["q"], kv, inp["kv_win"], inp["sinks"], m=m,
                                      w=0, rope_dims=wl.r)
    assert torch.count_nonzero(out[0, : m - 1]) == 0
    rows = np.array([m - 1, m, 300, 511])
    ref = O.prefill_attention("hca", npy(inp["q"][0]), npy(kv[0]), npy(inp["kv_win"][0]),
                              npy(inp["sinks"]), m=m, w=0, r=wl.r, rows=rows)
    check_close(npy(out[0, rows]), ref, "bf16", "hca w=0")
    assert api.device_error() == 0


@pytest.mark.parametrize("n,w", [(16384 + 37, 128), (8192 + 5, 64), (600, 64)])
def test_prefill_hca_64_heads_512_dims(n, w):
    """HCA prefill at the 64-head / 512-dim shape (m' = 128), including
    queries with no visible entry yet, a partial window and a ragged tail
    (the two larger cases run on the tensor cores, the smallest on CUDA cores)."""
    wl = synth.Workload(**{**synth.WORKLOADS["csa_prefill_128k"].__dict__, "kind": "hca", "w": w})
    inp, kv, m = _prefill_layer(wl, n, 2)
    out = api.compressed_attn_prefill("hca", inp["q"], kv, inp["kv_win"], inp["sinks"], m=m,
                                      w=wl.w, rope_dims=wl.r, q_gain=inp["q_gain"],
                                      kv_gain=inp["kv_gain"])
    for b in range(2):
        rows = _sample(n, [0, 1, 126, 127, 128, 255, 256, n - 1], seed=10 + b, count=10)
        ref = _oracle_rows("hca", inp, kv, None, wl, m, b, rows)
        check_close(npy(out[b, rows]), ref, "bf16", f"hca64 b={b}")
    assert api.device_error() == 0


def _gain(name, d, seed):
    """A non-unit RMSNorm gain, 1 + 0.1 N(0, 1) per dim."""
    return 1.0 + synth.Draw(seed, DEV).normal(name, (d,), 0.1)


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_prefill_tc_non_unit_gains(kind):
    """Non-unit query and KV gains on the tensor-core path (H = 64, d = 512):
    the query prologue multiplies q by its gain before RoPE (a separate branch
    from the all-ones one), the compressor and the window rows use the KV gain."""
    wl = synth.Workload(**{**synth.WORKLOADS["csa_prefill_128k"].__dict__, "kind": kind})
    n = 4096 + 3 if kind == "csa" else 2048 + 5
    inp = synth.prefill_inputs(wl, DEV, n=n, B=1)
    inp["q_gain"] = _gain("q_gain", wl.d, 21)
    inp["kv_gain"] = _gain("kv_gain", wl.d, 22)
    kvi = inp["kv"]
    m = wl.m if kind == "csa" else wl.m_hca
    idx = None
    if kind == "csa":
        kv = api.csa_compress(kvi["a"], kvi["b"], kvi["za"], kvi["zb"], kvi["bias_a"],
                              kvi["bias_b"], m, gain=inp["kv_gain"], rope_dims=wl.r)
        ik = inp["ik"]
        kI = api.csa_compress(ik["a"], ik["b"], ik["za"], ik["zb"], ik["bias_a"], ik["bias_b"], m,
                              rms_norm=False)
        q_pos = torch.arange(n, device=DEV, dtype=torch.int32)[None]
        idx = api.indexer_topk(inp["qI"], inp["w"], kI, q_pos, m, wl.k)
    else:
        kv = api.hca_compress(kvi["a"], kvi["za"], kvi["bias_a"], m, gain=inp["kv_gain"],
                              rope_dims=wl.r)
    # the compressor rows against the oracle's, gain included
    from tests.helpers import oracle_compress
    ents = [0, 1, kv.shape[1] // 2, kv.shape[1] - 1]
    check_close(npy(kv[0, ents]), oracle_compress(kind, kvi, m, 0, ents, True, inp["kv_gain"], wl.r),
                "bf16", "compress gain")
    out = api.compressed_attn_prefill(kind, inp["q"], kv, inp["kv_win"], inp["sinks"], m=m,
                                      w=wl.w, rope_dims=wl.r, idx=idx, q_gain=inp["q_gain"],
                                      kv_gain=inp["kv_gain"])
    rows = _sample(n, [0, 3, 4, 127, 128, m - 1, m, n - 1], seed=5, count=12)
    ref = _oracle_rows(kind, inp, kv, idx, wl, m, 0, rows)
    check_close(npy(out[0, rows]), ref, "bf16", f"{kind} prefill gains")
    assert api.device_error() == 0


@pytest.mark.slow
def test_prefill_csa_128k_full_size_sampled():
    """csa_prefill_128k at its full size (n = 131,072, the layer bench.py
    times): both compressors, indexer top-k and attention on the GPU; 64
    seeded sampled queries checked against the oracle -- queries with fewer
    visible entries than k (t < 4,096), rows of 16,384 < v <= 32,768 visible
    entries, block boundaries and t = n - 1.  Top-k sets under the tie-band
    rule; outputs with the oracle on the GPU's own index set."""
    from tests.helpers import check_topk
    wl = synth.WORKLOADS["csa_prefill_128k"]
    n = wl.n
    inp, kv, m = _prefill_layer(wl, n, 1)
    ik = inp["ik"]
    kI = api.csa_compress(ik["a"], ik["b"], ik["za"], ik["zb"], ik["bias_a"], ik["bias_b"], m,
                          rms_norm=False)
    q_pos = torch.arange(n, device=DEV, dtype=torch.int32)[None]
    idx = api.indexer_topk(inp["qI"], inp["w"], kI, q_pos, m, wl.k)
    out = api.compressed_attn_prefill("csa", inp["q"], kv, inp["kv_win"], inp["sinks"], m=m,
                                      w=wl.w, rope_dims=wl.r, idx=idx, q_gain=inp["q_gain"],
                                      kv_gain=inp["kv_gain"])
    torch.cuda.synchronize()
    rng = np.random.default_rng(2)
    fixed = [0, 3, 4, 4095, 4096, 4 * wl.k - 1, 4 * wl.k, 65535, 65536, 65539, n - 2, n - 1]
    rows = np.unique(np.r_[fixed, rng.integers(0, 4096, 12), rng.integers(65536, n, 30),
                           rng.integers(4096, 65536, 10)])[:64]
    KI = npy(kI[0])
    for t in rows:
        v = O.n_visible(int(t), m)
        s = O.indexer_scores(npy(inp["qI"][0, t]), npy(inp["w"][0, t]), KI[:v])
        check_topk(npy(idx[0, t]), s, wl.k, f"t={t}")
    ref = _oracle_rows("csa", inp, kv, idx, wl, m, 0, rows)
    check_close(npy(out[0, rows]), ref, "bf16", "csa prefill 128k")
    assert api.device_error() == 0


@pytest.mark.parametrize("n,w,m", [(8192 + 3, 128, 128), (1000, 64, 128), (261, 5, 16), (130, 128, 32)])
def test_prefill_hca_16_heads_128_dims_tensor_cores(n, w, m):
    """The 16-head / 128-dim HCA shape (hca_8k_bf16's heads) on the tensor
    cores: four queries per work item, so ragged tails (n not a multiple of
    4), blocks whose last query sees one more entry than the first, windows
    shorter than the block span and non-unit gains are all covered."""
    wl = synth.Workload(**{**synth.WORKLOADS["hca_8k_bf16"].__dict__, "w": w, "m_hca": m})
    inp, kv, _ = _prefill_layer(wl, n, 2)
    inp["q_gain"] = _gain("q_gain16", wl.d, 23)
    out = api.compressed_attn_prefill("hca", inp["q"], kv, inp["kv_win"], inp["sinks"], m=m,
                                      w=wl.w, rope_dims=wl.r, q_gain=inp["q_gain"],
                                      kv_gain=inp["kv_gain"])
    for b in range(2):
        rows = _sample(n, [0, 1, 2, 3, m - 2, m - 1, m, 4 * (m // 4) + 3, n - 4, n - 3, n - 2, n - 1],
                       seed=40 + b, count=16)
        ref = _oracle_rows("hca", inp, kv, None, wl, m, b, rows)
        check_close(npy(out[b, rows]), ref, "bf16", f"hca16 n={n} w={w} m={m} b={b}")
    assert api.device_error() == 0
