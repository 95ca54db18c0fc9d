"""One decode_1m layer (or one reduced csa_prefill_128k layer), repeated, for
a profiler to capture.

    python -m long_context_compressed_overlapped_b200.profile_case csa --calls 4
    python -m long_context_compressed_overlapped_b200.profile_case hca --calls 4
    python -m long_context_compressed_overlapped_b200.profile_case csa_fp8kv --calls 4
    python -m long_context_compressed_overlapped_b200.profile_case indexer --calls 4
    python -m long_context_compressed_overlapped_b200.profile_case indexer_256k --calls 4
    python -m long_context_compressed_overlapped_b200.profile_case compress --calls 4
    python -m long_context_compressed_overlapped_b200.profile_case prefill --calls 2
    python -m long_context_compressed_overlapped_b200.profile_case prefill_tail --calls 2

``csa``: one CSA decode layer through ``compressed_attn_decode`` (indexer with
e4m3 keys, top-k select, attention, combine); ``hca``: one HCA decode layer
(attention, combine); ``csa_fp8kv`` / ``hca_fp8kv``: the same layers with FP8
KV cache rows (decode_1m_fp8kv: 640-byte rows of e4m3 codes, bf16 RoPE dims
and fp32 scales); ``indexer``: ``indexer_topk`` on the CSA layer's indexer
inputs; ``indexer_256k``: the same on the decode_256k CSA layer (eight
sequences at a 262,144-token context, 65,536 bf16 indexer keys each, 134 MB,
routed by the bf16 indexer); ``compress``: ``decode_compress`` of the CSA layer with the new token at
position 1,048,575, which completes a block (ring store, window row, pooled
entry and e4m3 indexer key).  Four sequences at a 1,048,576-token context: 262,144 CSA entries
(1 GB of bf16 rows, 134 MB of e4m3 indexer keys) or 8,192 HCA entries per
sequence; about 1.3 GB on the device.  Inputs are the seeded synthetic draw of
the decode_1m workload.  ``prefill``: the csa_prefill_128k layer's shapes
(64 heads of 512 dims, 64 indexer heads of 128 dims, top-1,024, window 128)
at n = 16,384 tokens: both compressors, indexer_topk (the tensor-core
indexer over 4-query tiles, then the row top-k) and compressed_attn_prefill;
about 3 GB on the device.  ``prefill_tail``: indexer_topk for the last 16,384
queries of csa_prefill_128k (positions 114,688 .. 131,071 against the layer's
32,768 indexer keys: the longest score rows, 28,673 .. 32,768 entries);
about 2.3 GB on the device.  The process exits non-zero if a bounded device
wait gave up.
"""

import argparse
import ctypes as C
import sys

import torch

from . import api, native, runtime, synth


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("case", choices=("csa", "hca", "csa_fp8kv", "hca_fp8kv", "indexer", "indexer_256k", "compress",
                                        "prefill", "prefill_tail"))
    ap.add_argument("--calls", type=int, default=4)
    a = ap.parse_args(argv)
    if a.case == "prefill":
        return prefill_case(a.calls)
    if a.case == "prefill_tail":
        return prefill_tail_case(a.calls)
    wl = synth.WORKLOADS["decode_1m_fp8kv" if a.case.endswith("_fp8kv") else
                         "decode_256k" if a.case.endswith("_256k") else "decode_1m"]
    kind = "hca" if a.case.startswith("hca") else "csa"
    ctx = wl.ctx - 1 if a.case == "compress" else wl.ctx
    L = synth.decode_inputs(wl, "cuda", ctx=ctx, B=wl.B, layers=(kind,))[0]
    cargs = runtime.compress_args(wl, L) if a.case == "compress" else None
    for _ in range(a.calls):
        if a.case == "compress":
            native.check(native.lib().decode_compress(C.byref(cargs[0]), torch.cuda.current_stream().cuda_stream),
                         "decode_compress")
        elif a.case in ("indexer", "indexer_256k"):
            api.indexer_topk(L["qI"][:, None], L["w"][:, None], L["kI"], L["pos"][:, None], L["m"], wl.k,
                             kI_scale=L["kI_scale"])
        else:
            kw = dict(m=L["m"], rope_dims=wl.r, q_gain=L["q_gain"])
            if kind == "csa":
                kw.update(k=wl.k, qI=L["qI"], wI=L["w"], kI=L["kI"], kI_scale=L["kI_scale"])
            api.compressed_attn_decode(kind, L["q"], L["pos"], L["kv"], L["win"], L["sinks"], **kw)
    torch.cuda.synchronize()
    err = api.device_error()
    print(f"profile_case {a.case}: {a.calls} calls, device error {err}")
    return 1 if err else 0


def prefill_case(calls: int, n: int = 16384) -> int:
    wl = synth.WORKLOADS["csa_prefill_128k"]
    inp = synth.prefill_inputs(wl, "cuda", n=n)
    kvi, ik = inp["kv"], inp["ik"]
    q_pos = torch.arange(n, device="cuda", dtype=torch.int32)[None]
    for _ in range(calls):
        kv = api.csa_compress(kvi["a"], kvi["b"], kvi["za"], kvi["zb"], kvi["bias_a"], kvi["bias_b"], wl.m,
                              gain=inp["kv_gain"], rope_dims=wl.r)
        kI = api.csa_compress(ik["a"], ik["b"], ik["za"], ik["zb"], ik["bias_a"], ik["bias_b"], wl.m,
                              rms_norm=False)
        idx = api.indexer_topk(inp["qI"], inp["w"], kI, q_pos, wl.m, wl.k)
        api.compressed_attn_prefill("csa", inp["q"], kv, inp["kv_win"], inp["sinks"], m=wl.m, w=wl.w,
                                    rope_dims=wl.r, idx=idx, q_gain=inp["q_gain"], kv_gain=inp["kv_gain"])
    torch.cuda.synchronize()
    err = api.device_error()
    print(f"profile_case prefill (n={n}): {calls} calls, device error {err}")
    return 1 if err else 0


def prefill_tail_case(calls: int, nq: int = 16384) -> int:
    wl = synth.WORKLOADS["csa_prefill_128k"]
    D = synth.Draw(wl.seed + 100, "cuda")
    N = wl.n // wl.m
    qI = D.normal("qI", (1, nq, wl.HI, wl.dI), 1.0, torch.bfloat16)
    w = D.normal("w", (1, nq, wl.HI), 1.0 / wl.HI ** 0.5)
    kI = D.normal("kI", (1, N, wl.dI), 1.0, torch.bfloat16)
    q_pos = torch.arange(wl.n - nq, wl.n, device="cuda", dtype=torch.int32)[None]
    for _ in range(calls):
        api.indexer_topk(qI, w, kI, q_pos, wl.m, wl.k)
    torch.cuda.synchronize()
    err = api.device_error()
    print(f"profile_case prefill_tail ({nq} queries, {N} keys): {calls} calls, device error {err}")
    return 1 if err else 0


if __name__ == "__main__":
    sys.exit(main())
