"""GPU parity of compressed_attn_decode (one decode step per layer; CSA with
the lightning-indexer top-k, HCA dense; window ring and sink) against the
float64 oracle ("Paper Breakdown: DeepSeek-V4", section 4; "How DeepSeek-V4
architecture and training work together", "Two compressed views of one
history": interleaved CSA / HCA layers, top-1,024 and a 128-token window)."""

import pytest
import torch

from long_context_compressed_overlapped_b200 import api, synth
from oracle import csahca_oracle as O
from tests.helpers import check_close, check_topk, npy

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _decode_layer(L, wl, idx_out=None, idx_in=None):
    kw = dict(m=L["m"], rope_dims=wl.r, q_gain=L["q_gain"])
    if L["kind"] == "csa":
        kw.update(k=wl.k, qI=L["qI"], wI=L["w"], kI=L["kI"], kI_scale=L["kI_scale"],
                  idx_out=idx_out, idx_in=idx_in)
    return api.compressed_attn_decode(L["kind"], L["q"], L["pos"], L["kv"], L["win"], L["sinks"],
                                      **kw)


def _check_layer(L, wl, out, idx, seqs):
    for b in seqs:
        pos = int(L["pos"][b])
        sel = None
        if L["kind"] == "csa":
            v = min(O.n_visible(pos, L["m"]), L["kv"].shape[1])
            if L["kI_scale"] is not None:
                K = O.dequant_e4m3_rows(npy(L["kI"][b, :v]), npy(L["kI_scale"][b, :v]))
            else:
                K = npy(L["kI"][b, :v])
            s = O.indexer_scores(npy(L["qI"][b]), npy(L["w"][b]), K)
            check_topk(npy(idx[b]), s, wl.k, f"{L['kind']} b={b}")
            sel = npy(idx[b])
        ref = O.decode_attention(L["kind"], npy(L["q"][b]), pos, npy(L["kv"][b]), npy(L["win"][b]),
                                 npy(L["sinks"]), m=L["m"], w=wl.w, r=wl.r,
                                 q_gain=npy(L["q_gain"]), sel=sel)
        check_close(npy(out[b]), ref, wl.dtype, f"{L['kind']} b={b}")


@pytest.mark.parametrize("wl_name,ctx", [("decode_256k", 16384 + 7), ("decode_1m", 32768 + 130)])
def test_decode_layers(wl_name, ctx):
    """Interleaved layers of decode_256k (bf16 keys) and decode_1m (e4m3
    keys) at reduced context, positions including a ragged block tail."""
    wl = synth.WORKLOADS[wl_name]
    layers = synth.decode_inputs(wl, DEV, ctx=ctx, B=2)
    for L in layers:
        L["pos"] = torch.tensor([ctx, ctx - 200], device=DEV, dtype=torch.int32)
        idx = torch.empty(2, wl.k, dtype=torch.int32, device=DEV) if L["kind"] == "csa" else None
        out = _decode_layer(L, wl, idx_out=idx)
        _check_layer(L, wl, out, idx, range(2))
    assert api.device_error() == 0


def test_decode_short_context_edges():
    """pos < m - 1 (no entry visible), pos < w (partial window), visible <= k."""
    wl = synth.WORKLOADS["decode_256k"]
    layers = synth.decode_inputs(wl, DEV, ctx=4096, B=4)
    for L in layers:
        L["pos"] = torch.tensor([0, 2, 100, 4095], device=DEV, dtype=torch.int32)
        idx = torch.empty(4, wl.k, dtype=torch.int32, device=DEV) if L["kind"] == "csa" else None
        out = _decode_layer(L, wl, idx_out=idx)
        _check_layer(L, wl, out, idx, range(4))
    assert api.device_error() == 0


def test_decode_tiny_f32():
    """tiny_csa_f32 head shapes in fp32: tolerance 1e-5."""
    wl = synth.WORKLOADS["tiny_csa_f32"]
    wl = synth.Workload(**{**wl.__dict__, "layers": ("csa", "hca"), "m_hca": 16})
    layers = synth.decode_inputs(wl, DEV, ctx=512, B=2)
    for L in layers:
        L["pos"] = torch.tensor([511, 300], device=DEV, dtype=torch.int32)
        idx = torch.empty(2, wl.k, dtype=torch.int32, device=DEV) if L["kind"] == "csa" else None
        out = _decode_layer(L, wl, idx_out=idx)
        _check_layer(L, wl, out, idx, range(2))
    assert api.device_error() == 0


def test_decode_idx_in_matches_internal_selection():
    wl = synth.WORKLOADS["decode_256k"]
    L = synth.decode_inputs(wl, DEV, ctx=8192, B=2, layers=("csa",))[0]
    idx = torch.empty(2, wl.k, dtype=torch.int32, device=DEV)
    out1 = _decode_layer(L, wl, idx_out=idx)
    out2 = _decode_layer(L, wl, idx_in=idx)
    assert torch.equal(out1, out2)
    assert api.device_error() == 0


@pytest.mark.slow
def test_decode_1m_full_size_one_sequence_checked():
    """decode_1m at full context (1,048,576 tokens, 262,144 CSA entries with
    e4m3 keys, 8,192 HCA entries), all four layers; sequence 0 checked."""
    wl = synth.WORKLOADS["decode_1m"]
    layers = synth.decode_inputs(wl, DEV)
    for L in layers:
        idx = torch.empty(wl.B, wl.k, dtype=torch.int32, device=DEV) if L["kind"] == "csa" else None
        out = _decode_layer(L, wl, idx_out=idx)
        _check_layer(L, wl, out, idx, [0])
    assert api.device_error() == 0


@pytest.mark.parametrize("wl_name", ["decode_256k", "decode_1m"])
def test_decode_non_unit_query_gain(wl_name):
    """A non-unit query gain (1 + 0.1 N(0, 1) per dim) on the tensor-core
    decode path of both layer kinds: the prologue multiplies q by the gain
    before RoPE and takes the RMS from the raw values."""
    wl = synth.WORKLOADS[wl_name]
    layers = synth.decode_inputs(wl, DEV, ctx=16384 + 3, B=2)
    for li, L in enumerate(layers):
        L["q_gain"] = 1.0 + synth.Draw(30 + li, DEV).normal("q_gain", (wl.d,), 0.1)
        idx = torch.empty(2, wl.k, dtype=torch.int32, device=DEV) if L["kind"] == "csa" else None
        out = _decode_layer(L, wl, idx_out=idx)
        _check_layer(L, wl, out, idx, range(2))
    assert api.device_error() == 0


def test_decode_large_value_rows():
    """Cache and window rows scaled by 1e5 (finite in bf16, far beyond fp16's
    65,504): the split partials must stay finite and the output match the
    oracle (compared after dividing both by the scale, with the bf16
    tolerances).  A query gain of 1e-5 keeps the scores at their usual size,
    so the softmax weights are as in an unscaled layer and only the values
    are large."""
    wl = synth.WORKLOADS["decode_256k"]
    scale = 1e5
    layers = synth.decode_inputs(wl, DEV, ctx=8192 + 5, B=2)
    for L in layers:
        L["kv"] = (L["kv"].float() * scale).to(torch.bfloat16)
        L["win"] = (L["win"].float() * scale).to(torch.bfloat16)
        L["q_gain"] = torch.full((wl.d,), 1.0 / scale, device=DEV)
        idx = torch.empty(2, wl.k, dtype=torch.int32, device=DEV) if L["kind"] == "csa" else None
        out = _decode_layer(L, wl, idx_out=idx)
        assert torch.isfinite(out.float()).all(), f"{L['kind']}: non-finite output"
        for b in range(2):
            pos = int(L["pos"][b])
            sel = npy(idx[b]) if idx is not None else None
            ref = O.decode_attention(L["kind"], npy(L["q"][b]), pos, npy(L["kv"][b]), npy(L["win"][b]),
                                     npy(L["sinks"]), m=L["m"], w=wl.w, r=wl.r,
                                     q_gain=npy(L["q_gain"]), sel=sel)
            check_close(npy(out[b]) / scale, ref / scale, "bf16", f"{L['kind']} x1e5 b={b}")
    assert api.device_error() == 0


@pytest.mark.slow
def test_decode_256k_full_size_all_sequences():
    """decode_256k at its full size: B = 8 sequences at a 262,144-token
    context (65,536 CSA entries with bf16 indexer keys, 2,048 HCA entries),
    one CSA and one HCA layer; every sequence checked."""
    wl = synth.WORKLOADS["decode_256k"]
    layers = synth.decode_inputs(wl, DEV)
    for L in layers:
        idx = torch.empty(wl.B, wl.k, dtype=torch.int32, device=DEV) if L["kind"] == "csa" else None
        out = _decode_layer(L, wl, idx_out=idx)
        _check_layer(L, wl, out, idx, range(wl.B))
    assert api.device_error() == 0


def _fp8_kv_rows(L, wl, b):
    """The rows an FP8 KV cache of layer L stands for (sequence b), float64."""
    return O.dequant_kv_rows_fp8(*(npy(t) for t in synth.unpack_kv_rows_fp8(L["kv"][b], wl.d, wl.r)))


@pytest.mark.parametrize("ctx,B", [(32768 + 130, 2), (4096, 4)])
def test_decode_fp8_kv_layers(ctx, B):
    """decode_1m with FP8 KV cache rows (e4m3 non-RoPE dims with one fp32
    scale per 64, bf16 RoPE dims), CSA and HCA layers: the attention reads the
    rows the cache stands for (the oracle dequantises them); gathered (CSA)
    and contiguous (HCA) rows, a ragged block tail and partial windows."""
    wl = synth.WORKLOADS["decode_1m_fp8kv"]
    layers = synth.decode_inputs(wl, DEV, ctx=ctx, B=B, layers=("csa", "hca"))
    for L in layers:
        assert L["kv"].dtype == torch.uint8
        L["pos"] = torch.tensor([ctx, ctx - 200, 100, 7][:B], device=DEV, dtype=torch.int32)
        idx = torch.empty(B, wl.k, dtype=torch.int32, device=DEV) if L["kind"] == "csa" else None
        out = _decode_layer(L, wl, idx_out=idx)
        for b in range(B):
            pos = int(L["pos"][b])
            sel = None
            if L["kind"] == "csa":
                v = min(O.n_visible(pos, L["m"]), L["kv"].shape[1])
                K = O.dequant_e4m3_rows(npy(L["kI"][b, :v]), npy(L["kI_scale"][b, :v]))
                check_topk(npy(idx[b]), O.indexer_scores(npy(L["qI"][b]), npy(L["w"][b]), K), wl.k,
                           f"fp8kv b={b}")
                sel = npy(idx[b])
            ref = O.decode_attention(L["kind"], npy(L["q"][b]), pos, _fp8_kv_rows(L, wl, b), npy(L["win"][b]),
                                     npy(L["sinks"]), m=L["m"], w=wl.w, r=wl.r, q_gain=npy(L["q_gain"]),
                                     sel=sel)
            check_close(npy(out[b]), ref, "bf16", f"fp8kv {L['kind']} b={b} pos={pos}")
    assert api.device_error() == 0


@pytest.mark.slow
def test_decode_fp8_kv_full_size():
    """decode_1m_fp8kv at the full 1,048,576-token context, all four layers,
    sequence 0 checked."""
    wl = synth.WORKLOADS["decode_1m_fp8kv"]
    layers = synth.decode_inputs(wl, DEV)
    for L in layers:
        idx = torch.empty(wl.B, wl.k, dtype=torch.int32, device=DEV) if L["kind"] == "csa" else None
        out = _decode_layer(L, wl, idx_out=idx)
        pos = int(L["pos"][0])
        sel = npy(idx[0]) if idx is not None else None
        ref = O.decode_attention(L["kind"], npy(L["q"][0]), pos, _fp8_kv_rows(L, wl, 0), npy(L["win"][0]),
                                 npy(L["sinks"]), m=L["m"], w=wl.w, r=wl.r, q_gain=npy(L["q_gain"]), sel=sel)
        check_close(npy(out[0]), ref, "bf16", f"fp8kv full {L['kind']}")
    assert api.device_error() == 0
