"""GPU parity of decode_compress, one decode step of a layer's compressors,
against the float64 oracle.  The step puts the new token's streams in the
ring and writes its window row.  When the token completes a block it also
writes the new CSA / HCA entry and the indexer key ("Paper Breakdown:
DeepSeek-V4", section 4: CSA KV Compression, HCA, Sliding window KV,
Additional Techniques).  Also covered: the decode step bench.py times
(compressors, indexer, top-k, attention per layer, replayed as a CUDA graph)
against the oracle's decode step."""

import ctypes as C

import numpy as np
import pytest
import torch

import bench
from long_context_compressed_overlapped_b200 import api, native, runtime, synth
from oracle import csahca_oracle as O
from tests.helpers import check_close, check_topk, npy

pytestmark = pytest.mark.gpu
DEV = "cuda"
NAMES = {"csa": ("a", "b", "za", "zb"), "hca": ("a", "za")}


def _replay(wl, kind, n, B, lags, gain):
    """Decode every token of a stream from position 0, one decode_compress
    call per step; sequence b takes token t - lags[b] at step t."""
    m = wl.m if kind == "csa" else wl.m_hca
    wl = synth.Workload(**{**wl.__dict__, "kind": kind})
    inp = synth.prefill_inputs(wl, DEV, n=n, B=B)
    names = NAMES[kind]
    R = 2 * m if kind == "csa" else m
    dt, d, w = wl.torch_dtype, wl.d, wl.w
    st = dict(ring=torch.zeros(B, R, len(names), d, dtype=dt, device=DEV),
              kv=torch.zeros(B, n // m, d, dtype=dt, device=DEV),
              win=torch.zeros(B, w, d, dtype=dt, device=DEV))
    if kind == "csa":
        st["iring"] = torch.zeros(B, R, 4, wl.dI, dtype=dt, device=DEV)
        st["kI"] = torch.zeros(B, n // m, wl.dI, dtype=dt, device=DEV)
    ar = torch.arange(B, device=DEV)
    for t in range(n + max(lags)):
        p = [t - lag for lag in lags]
        tok = torch.tensor([min(max(x, 0), n - 1) for x in p], device=DEV)
        pos = torch.tensor([x if 0 <= x < n else -1 for x in p], dtype=torch.int32, device=DEV)
        streams = tuple(inp["kv"][s_][ar, tok].contiguous() for s_ in names)
        kw = {}
        if kind == "csa":
            kw = dict(istreams=tuple(inp["ik"][s_][ar, tok].contiguous() for s_ in names),
                      ibias_a=inp["ik"]["bias_a"], ibias_b=inp["ik"]["bias_b"], iring=st["iring"],
                      kI=st["kI"])
        api.decode_compress(kind, pos, streams, st["ring"], st["kv"], m=m, bias_a=inp["kv"]["bias_a"],
                            bias_b=inp["kv"].get("bias_b"), kv_raw=inp["kv_win"][ar, tok].contiguous(),
                            win=st["win"], kv_gain=gain, rope_dims=wl.r, **kw)
    torch.cuda.synchronize()
    return wl, inp, st, m


def _check_replay(wl, kind, inp, st, m, n, B, gain):
    names = NAMES[kind]
    R = 2 * m if kind == "csa" else m
    g = npy(gain)
    for b in range(B):
        s = {s_: npy(inp["kv"][s_][b]) for s_ in names}
        if kind == "csa":
            pooled = O.csa_pool(s["a"], s["b"], s["za"], s["zb"], npy(inp["kv"]["bias_a"]),
                                npy(inp["kv"]["bias_b"]), m)
            ik = {s_: npy(inp["ik"][s_][b]) for s_ in names}
            keys = O.csa_pool(ik["a"], ik["b"], ik["za"], ik["zb"], npy(inp["ik"]["bias_a"]),
                              npy(inp["ik"]["bias_b"]), m)
            check_close(npy(st["kI"][b]), keys, wl.dtype, f"indexer keys b={b}")
        else:
            pooled = O.hca_pool(s["a"], s["za"], npy(inp["kv"]["bias_a"]), m)
        rows = O.finish_rows(pooled, np.arange(pooled.shape[0]) * m, g, wl.r)
        check_close(npy(st["kv"][b]), rows, wl.dtype, f"{kind} entries b={b}")
        p = np.arange(n - wl.w, n)
        wrows = O.finish_rows(npy(inp["kv_win"][b, p]), p, g, wl.r)
        check_close(npy(st["win"][b, p % wl.w]), wrows, wl.dtype, f"window b={b}")
        p = np.arange(n - R, n)
        for j, s_ in enumerate(names):         # the ring holds the last R raw tokens, bit for bit
            assert torch.equal(st["ring"][b, p % R, j], inp["kv"][s_][b, p])


def test_decode_compress_tiny_csa_f32():
    """tiny_csa_f32 shapes (d 64, r 16, m 4, d_I 32, w 16) in fp32, 40 tokens
    replayed one call per step, the second sequence 5 tokens behind."""
    wl = synth.WORKLOADS["tiny_csa_f32"]
    gain = 1 + 0.1 * torch.randn(wl.d, generator=torch.Generator().manual_seed(5)).to(DEV)
    wl, inp, st, m = _replay(wl, "csa", 40, 2, [0, 5], gain)
    _check_replay(wl, "csa", inp, st, m, 40, 2, gain)
    assert api.device_error() == 0


def test_decode_compress_hca_bf16():
    """hca_8k_bf16 shapes (d 128, r 64, m' 128, w 128): 300 tokens (two
    entries and a ragged tail), the second sequence 45 tokens behind."""
    wl = synth.WORKLOADS["hca_8k_bf16"]
    gain = torch.ones(wl.d, device=DEV)
    wl, inp, st, m = _replay(wl, "hca", 300, 2, [0, 45], gain)
    _check_replay(wl, "hca", inp, st, m, 300, 2, gain)
    assert api.device_error() == 0


def _check_e4m3_key(codes, scales, key, what):
    """codes/scales from the GPU; key: the oracle's pooled fp64 row.  The
    scale must be the row's amax / 448 and each code a nearest e4m3 of
    key / scale (a neighbour only where the two are equally near within the
    fp32 error of the pooling)."""
    amax = np.abs(key.reshape(-1, 128)).max(axis=1)
    np.testing.assert_allclose(scales, amax / 448.0, rtol=1e-5, err_msg=what)
    xs = key / np.repeat(scales.astype(np.float64), 128)
    want = O.e4m3_encode(xs)
    d_got = np.abs(O.e4m3_decode(codes) - xs)
    d_want = np.abs(O.e4m3_decode(want) - xs)
    assert (d_got <= d_want + 1e-4 * np.maximum(np.abs(xs), 1e-3)).all(), what
    assert (codes == want).mean() >= 0.99, what


def test_decode_compress_decode_1m_shapes():
    """decode_1m shapes (B 4, d 512, d_I 128 e4m3, m 4, m' 128, w 128), one
    call per layer with the rings as drawn, at positions that complete a
    block near 2^20, complete none, complete the first block, and complete
    block N-2."""
    wl = synth.WORKLOADS["decode_1m"]
    ctx = (1 << 20) - 1
    layers = synth.decode_inputs(wl, DEV, ctx=ctx, layers=("csa", "hca"))
    for L in layers:
        m = L["m"]
        L["pos"] = torch.tensor([ctx, ctx - 1, m - 1, ctx - m], dtype=torch.int32, device=DEV)
        host = {k_: (v.cpu().clone() if isinstance(v, torch.Tensor) else v) for k_, v in L.items()}
        args, keep = runtime.compress_args(wl, L)
        native.check(native.lib().decode_compress(C.byref(args), torch.cuda.current_stream().cuda_stream),
                     "decode_compress")
        torch.cuda.synchronize()
        csa = L["kind"] == "csa"
        names = NAMES[L["kind"]]
        cols = ("ca", "cb", "cza", "czb") if csa else ("ca", "cza")
        R = 2 * m if csa else m
        for b in range(wl.B):
            pos = int(host["pos"][b])
            ring = {s_: npy(host["ring"][b, :, j]) for j, s_ in enumerate(names)}
            new = {s_: npy(host[c_][b]) for s_, c_ in zip(names, cols)}
            biases = (npy(host["bias_a"]), npy(host["bias_b"]) if csa else None)
            _, entry, win_row = O.decode_compress_step(L["kind"], pos, new, ring, biases, m,
                                                       kv_raw=npy(host["kv_raw"][b]),
                                                       gain=npy(host["kv_gain"]), r=wl.r)
            what = f"{L['kind']} b={b} pos={pos}"
            check_close(npy(L["win"][b, pos % wl.w]), win_row, "bf16", what + " window")
            for j, c_ in enumerate(cols):
                assert torch.equal(L["ring"][b, pos % R, j].cpu(), host[c_][b]), what + " ring"
            emitted = (pos + 1) % m == 0
            assert (entry is not None) == emitted
            if emitted:
                i = entry[0]
                check_close(npy(L["kv"][b, i]), entry[2], "bf16", what + " entry")
                lo = max(i - 2, 0)
                assert torch.equal(L["kv"][b, lo:i].cpu(), host["kv"][b, lo:i]), what + " neighbours"
            else:
                i = (pos + 1) // m
                lo = max(i - 2, 0)
                assert torch.equal(L["kv"][b, lo:i + 1].cpu(), host["kv"][b, lo:i + 1]), what + " untouched"
            if csa and emitted:
                iring = {s_: npy(host["iring"][b, :, j]) for j, s_ in enumerate(names)}
                inew = {s_: npy(host[c_][b]) for s_, c_ in zip(names, ("ia", "ib", "iza", "izb"))}
                _, ient, _ = O.decode_compress_step("csa", pos, inew, iring,
                                                    (npy(host["ibias_a"]), npy(host["ibias_b"])), m,
                                                    normalize=False)
                _check_e4m3_key(npy(L["kI"][b, i]), npy(L["kI_scale"][b, i]), ient[1], what + " key")
        del keep
    assert api.device_error() == 0


def _check_fp8_kv_row(packed, finished, r, what):
    """An FP8 KV row written by decode_compress against the oracle's quantiser
    of the finished entry: RoPE dims within the bf16 tolerance, block scales
    amax / 448 to 1e-5 relative, and each code a nearest e4m3 of x / scale (a
    neighbour only where the two are equally near within the fp32 error of
    the pooling; at least 99 % identical)."""
    d = finished.shape[-1]
    codes, scales, rope = synth.unpack_kv_rows_fp8(packed, d, r)
    oc, osc, orope = O.quantize_kv_rows_fp8(finished, r)
    check_close(npy(rope), orope, "bf16", what + " rope dims")
    x = finished[: d - r]
    amax = np.abs(x.reshape(-1, 64)).max(axis=1)
    np.testing.assert_allclose(npy(scales), amax / 448.0, rtol=1e-5, err_msg=what)
    xs = x / np.repeat(npy(scales), 64)
    got = npy(codes)
    d_got = np.abs(O.e4m3_decode(got) - xs)
    d_want = np.abs(O.e4m3_decode(O.e4m3_encode(xs)) - xs)
    assert (d_got <= d_want + 1e-4 * np.maximum(np.abs(xs), 1e-3)).all(), what
    assert (got == oc).mean() >= 0.99, what


def test_decode_compress_fp8_kv_rows():
    """decode_compress into FP8 KV caches (decode_1m_fp8kv shapes): CSA and
    HCA layers at positions that complete a block (near 2^20, the first block,
    block N-2) and one that completes none; the new entry is stored as an FP8
    KV row and its neighbours are untouched."""
    wl = synth.WORKLOADS["decode_1m_fp8kv"]
    ctx = (1 << 20) - 1
    layers = synth.decode_inputs(wl, DEV, ctx=ctx, layers=("csa", "hca"))
    for L in layers:
        m = L["m"]
        L["pos"] = torch.tensor([ctx, ctx - 1, m - 1, ctx - m], dtype=torch.int32, device=DEV)
        host = {k_: (v.cpu().clone() if isinstance(v, torch.Tensor) else v) for k_, v in L.items()}
        args, keep = runtime.compress_args(wl, L)
        native.check(native.lib().decode_compress(C.byref(args), torch.cuda.current_stream().cuda_stream),
                     "decode_compress")
        torch.cuda.synchronize()
        csa = L["kind"] == "csa"
        names = NAMES[L["kind"]]
        cols = ("ca", "cb", "cza", "czb") if csa else ("ca", "cza")
        for b in range(wl.B):
            pos = int(host["pos"][b])
            ring = {s_: npy(host["ring"][b, :, j]) for j, s_ in enumerate(names)}
            new = {s_: npy(host[c_][b]) for s_, c_ in zip(names, cols)}
            biases = (npy(host["bias_a"]), npy(host["bias_b"]) if csa else None)
            _, entry, _ = O.decode_compress_step(L["kind"], pos, new, ring, biases, m,
                                                 kv_raw=npy(host["kv_raw"][b]), gain=npy(host["kv_gain"]), r=wl.r)
            what = f"fp8kv {L['kind']} b={b} pos={pos}"
            if entry is not None:
                i = entry[0]
                _check_fp8_kv_row(L["kv"][b, i].cpu(), entry[2], wl.r, what)
                lo = max(i - 2, 0)
                assert torch.equal(L["kv"][b, lo:i].cpu(), host["kv"][b, lo:i]), what + " neighbours"
            else:
                i = (pos + 1) // m
                assert torch.equal(L["kv"][b, max(i - 2, 0):i + 1].cpu(),
                                   host["kv"][b, max(i - 2, 0):i + 1]), what + " untouched"
        del keep
    assert api.device_error() == 0


def _check_bench_step(ctx, B, seqs, workload="decode_1m"):
    """The step bench.py times (per layer decode_compress then
    compressed_attn_decode, CSA, HCA, CSA, HCA, replayed as a CUDA graph)
    against the oracle's decode step for the sequences `seqs`.  Selections
    must pass the top-k tolerance and outputs are compared on the GPU's
    selections."""
    wl = synth.WORKLOADS[workload]
    layers = synth.decode_inputs(wl, DEV, ctx=ctx, B=B)
    host = bench.host_layers(layers)
    stream = torch.cuda.Stream()
    step = runtime.DecodeStep(wl, layers, stream, keep_idx=True)
    graph = runtime.DecodeGraph(step)
    with torch.cuda.stream(stream):
        for _ in range(3):
            graph()                              # replays leave the same state
    torch.cuda.synchronize()
    assert api.device_error(stream) == 0
    for b in seqs:
        scores = []
        bench.oracle_decode_sequence(wl, host, b, scores_out=scores)
        sels = [None if ix is None else npy(ix[b]) for ix in step.idx]
        si = iter(scores)
        for li, L in enumerate(layers):
            if L["kind"] == "csa":
                check_topk(sels[li], next(si), wl.k, f"layer {li} b={b}")
        ref = bench.oracle_decode_sequence(wl, host, b, sels=sels)
        for li, o in enumerate(step.outputs):
            check_close(npy(o[b]), ref[li], "bf16", f"layer {li} b={b}")


def test_bench_decode_step_from_host_buffers():
    """The end-to-end form of the step (runtime.HostIOGraph): the device input
    arena is cleared, the step's inputs arrive from pinned host memory layer
    by layer inside the graph, and the outputs read back into host memory
    match the oracle."""
    wl = synth.WORKLOADS["decode_1m"]
    ctx, B = (1 << 15) - 1, 2
    layers = synth.decode_inputs(wl, DEV, ctx=ctx, B=B)
    io = runtime.StepIO(layers, DEV)
    host = bench.host_layers(layers)
    host_in = io.inp.cpu().pin_memory()
    host_out = torch.zeros(io.out.shape, dtype=io.out.dtype).pin_memory()
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    step = runtime.DecodeStep(wl, layers, stream, keep_idx=True)
    with torch.cuda.stream(stream):
        step()                                   # the library's first-call set-up
    torch.cuda.synchronize()
    graph = runtime.HostIOGraph(step, io, host_in, host_out)
    io.inp.zero_()
    io.out.zero_()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        graph()
    torch.cuda.synchronize()
    assert api.device_error(stream) == 0
    assert torch.equal(io.inp.cpu(), host_in)
    for b in range(B):
        sels = [None if ix is None else npy(ix[b]) for ix in step.idx]
        ref = bench.oracle_decode_sequence(wl, host, b, sels=sels)
        for li, L in enumerate(layers):
            a, e = io.out_ranges[li]
            o = host_out[a:e].view(L["out"].dtype).view(L["out"].shape)
            check_close(npy(o[b]), ref[li], "bf16", f"host output, layer {li} b={b}")


def test_bench_decode_step_with_compressors():
    """At a 32,767-token context, where the new token completes a CSA and an
    HCA block; both sequences checked."""
    _check_bench_step((1 << 15) - 1, 2, range(2))


def test_bench_decode_step_fp8_kv():
    """The bench's step with FP8 KV caches at a 32,767-token context (the new
    token completes a CSA and an HCA block, stored as FP8 KV rows)."""
    _check_bench_step((1 << 15) - 1, 2, range(2), workload="decode_1m_fp8kv")


@pytest.mark.slow
def test_bench_decode_step_full_size():
    """decode_1m exactly as bench.py runs it: B = 4 at the full 1,048,576-token
    context (262,144 CSA entries with e4m3 keys, 8,192 HCA entries per
    sequence), the CUDA-graph step with compressors; sequence 0 checked."""
    _check_bench_step(synth.WORKLOADS["decode_1m"].ctx, 4, [0])


def test_decode_compress_options():
    """decode_256k shapes (bf16 indexer keys): no RMSNorm (RoPE only), no
    window row, and an entry past the cache's capacity (not stored); the
    second sequence's token completes block N_cap, the first's block
    N_cap - 1."""
    wl = synth.WORKLOADS["decode_256k"]
    ctx = 63
    L = synth.decode_inputs(wl, DEV, ctx=ctx, B=2, layers=("csa",))[0]
    m = L["m"]
    N_cap = L["kv"].shape[1]
    assert N_cap == (ctx + 1) // m
    L["pos"] = torch.tensor([ctx, ctx + m], dtype=torch.int32, device=DEV)
    host = {k_: (v.cpu().clone() if isinstance(v, torch.Tensor) else v) for k_, v in L.items()}
    names = NAMES["csa"]
    api.decode_compress("csa", L["pos"], tuple(L[c] for c in ("ca", "cb", "cza", "czb")), L["ring"], L["kv"],
                        m=m, bias_a=L["bias_a"], bias_b=L["bias_b"], kv_raw=None, win=None,
                        kv_gain=L["kv_gain"], kv_norm=False, rope_dims=wl.r,
                        istreams=tuple(L[c] for c in ("ia", "ib", "iza", "izb")), ibias_a=L["ibias_a"],
                        ibias_b=L["ibias_b"], iring=L["iring"], kI=L["kI"])
    torch.cuda.synchronize()
    assert torch.equal(L["win"].cpu(), host["win"])                 # no window row
    for b in range(2):
        pos = int(host["pos"][b])
        ring = {s_: npy(host["ring"][b, :, j]) for j, s_ in enumerate(names)}
        new = {s_: npy(host[c_][b]) for s_, c_ in zip(names, ("ca", "cb", "cza", "czb"))}
        _, entry, _ = O.decode_compress_step("csa", pos, new, ring, (npy(host["bias_a"]), npy(host["bias_b"])),
                                             m, r=wl.r, normalize=False)
        iring = {s_: npy(host["iring"][b, :, j]) for j, s_ in enumerate(names)}
        inew = {s_: npy(host[c_][b]) for s_, c_ in zip(names, ("ia", "ib", "iza", "izb"))}
        _, ient, _ = O.decode_compress_step("csa", pos, inew, iring, (npy(host["ibias_a"]), npy(host["ibias_b"])),
                                            m, normalize=False)
        i = entry[0]
        if i < N_cap:
            check_close(npy(L["kv"][b, i]), entry[2], "bf16", f"b={b} entry without norm")
            check_close(npy(L["kI"][b, i]), ient[1], "bf16", f"b={b} bf16 key")
            assert torch.equal(L["kv"][b, :i].cpu(), host["kv"][b, :i])
        else:                                                         # past the capacity: nothing stored
            assert torch.equal(L["kv"][b].cpu(), host["kv"][b])
            assert torch.equal(L["kI"][b].cpu(), host["kI"][b])
        for j, c_ in enumerate(("ca", "cb", "cza", "czb")):
            assert torch.equal(L["ring"][b, pos % (2 * m), j].cpu(), host[c_][b])
    assert api.device_error() == 0
