"""Torch-facing wrappers of the C-ABI entry points (same names).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, outputs and workspaces are allocated with torch when the caller
does not pass them, and the call goes to libcsahca.so on the current CUDA
stream.  Every step of the path runs in the library's kernels.
"""

from __future__ import annotations

import ctypes as C

import torch

from . import native as N

_DT = {torch.float32: N.F32, torch.bfloat16: N.BF16, torch.uint8: N.E4M3}


def _dt(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return _DT[t.dtype]


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the CUDA library must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the CUDA library must be contiguous")
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _f32(t):
    return None if t is None else t.contiguous().float()


def _compress(kind, a, za, bias_a, m, *, b=None, zb=None, bias_b=None, gain=None,
              rms_norm=True, rope_dims=0, rope_base=10000.0, eps=1e-6, first_block=0,
              num_blocks=-1, out=None, stream=None):
    B, n, c = a.shape
    nb = (n // m - first_block) if num_blocks < 0 else num_blocks
    if out is None:
        out = torch.empty(B, max(nb, 0), c, dtype=a.dtype, device=a.device)
    bias_a = _f32(bias_a)
    bias_b = _f32(bias_b)
    gain = _f32(gain)
    args = N.CompressArgs(dtype=_dt(a), B=B, n=n, c=c, m=m, first_block=first_block,
                          num_blocks=num_blocks, rms_norm=int(bool(rms_norm)),
                          rope_dims=rope_dims, rope_base=rope_base, eps=eps,
                          a=_ptr(a), b=_ptr(b), za=_ptr(za), zb=_ptr(zb), bias_a=_ptr(bias_a),
                          bias_b=_ptr(bias_b), gain=_ptr(gain), out=_ptr(out))
    fn = N.lib().csa_compress if kind == "csa" else N.lib().hca_compress
    N.check(fn(C.byref(args), _stream(stream)), f"{kind}_compress")
    return out


def csa_compress(a, b, za, zb, bias_a, bias_b, m, **kw):
    """Overlapped two-stream compression (ratio 1/m, 2m tokens per entry),
    then optional RMSNorm * gain and RoPE at position i*m.  [B, n, c] -> [B, n/m, c]."""
    return _compress("csa", a, za, bias_a, m, b=b, zb=zb, bias_b=bias_b, **kw)


def hca_compress(a, za, bias_a, m, **kw):
    """Non-overlapped single-stream compression (ratio 1/m'), then optional
    RMSNorm * gain and RoPE at position i*m'."""
    return _compress("hca", a, za, bias_a, m, **kw)


def indexer_topk(qI, w, kI, q_pos, m, k, *, kI_scale=None, idx=None, scores_out=None,
                 sel_scores=None, entry_base=0, stream=None):
    """Lightning-indexer scores over the visible compressed keys and the
    per-query top-k (ties to the lower index), sorted ascending, -1 padded.

    qI [B, nq, HI, dI]; w [B, nq, HI] f32; kI [B, N, dI] (f32/bf16, or uint8
    e4m3 codes with kI_scale [B, N, dI/128]); q_pos [B, nq] int32.
    Context parallelism: kI holds the global entries entry_base ..
    entry_base + N - 1 (idx then holds local rows), and sel_scores
    [B, nq, k] f32 receives the score of each selected row."""
    B, nq, HI, dI = qI.shape
    Nk = kI.shape[1]
    if idx is None:
        idx = torch.empty(B, nq, k, dtype=torch.int32, device=qI.device)
    w = _f32(w)
    q_pos = q_pos.to(torch.int32).contiguous()
    args = N.IndexerArgs(q_dtype=_dt(qI), k_dtype=_dt(kI), B=B, nq=nq, HI=HI, dI=dI, N=Nk, m=m,
                         k=k, qI=_ptr(qI), w=_ptr(w), kI=_ptr(kI),
                         kI_scale=_ptr(_f32(kI_scale)), q_pos=_ptr(q_pos), idx=_ptr(idx),
                         scores_out=_ptr(scores_out), sel_scores=_ptr(sel_scores),
                         entry_base=int(entry_base))
    L = N.lib()
    ws_bytes = L.csahca_indexer_workspace_size(C.byref(args))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=qI.device) if ws_bytes else None
    args.workspace = _ptr(ws)
    args.workspace_bytes = ws_bytes
    N.check(L.indexer_topk(C.byref(args), _stream(stream)), "indexer_topk")
    return idx


def compressed_attn_prefill(kind, q, kv_comp, kv_win, sinks, *, m, w, rope_dims, idx=None,
                            q_gain=None, kv_gain=None, q_norm=True, kv_norm=True,
                            rope_base=10000.0, eps=1e-6, scale=0.0, out=None, stream=None):
    """CSA (selected entries) or HCA (every visible entry) attention plus the
    sliding window and per-head sink, for every query of a prefill.

    q [B, n, H, d] raw; kv_comp [B, N, d] final rows; kv_win [B, n, d] raw
    per-token rows; idx [B, n, k] int32 (CSA)."""
    B, n, H, d = q.shape
    Nc = kv_comp.shape[1]
    if out is None:
        out = torch.empty_like(q)
    kk = idx.shape[2] if idx is not None else 0
    args = N.AttnArgs(kind=N.CSA if kind == "csa" else N.HCA, dtype=_dt(q), B=B, n=n, H=H, d=d,
                      N=Nc, m=m, k=kk, w=w, rope_dims=rope_dims, rope_base=rope_base, eps=eps,
                      scale=scale, q_norm=int(bool(q_norm)), kv_norm=int(bool(kv_norm)),
                      q=_ptr(q), kv_comp=_ptr(kv_comp) if Nc > 0 else None, kv_win=_ptr(kv_win),
                      q_gain=_ptr(_f32(q_gain)), kv_gain=_ptr(_f32(kv_gain)),
                      idx=_ptr(idx), sinks=_ptr(_f32(sinks)), out=_ptr(out))
    L = N.lib()
    ws_bytes = L.csahca_prefill_workspace_size(C.byref(args))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device) if ws_bytes else None
    args.workspace = _ptr(ws)
    args.workspace_bytes = ws_bytes
    N.check(L.compressed_attn_prefill(C.byref(args), _stream(stream)), "compressed_attn_prefill")
    return out


def decode_args(kind, q, pos, kv_cache, win, sinks, *, m, rope_dims, k=0, qI=None, wI=None,
                kI=None, kI_scale=None, idx_in=None, idx_out=None, q_gain=None, q_norm=True,
                rope_base=10000.0, eps=1e-6, scale=0.0, out=None, entry_base=0, partial_out=None,
                skip_window=False):
    """Build the DecodeArgs struct (and keep the tensors it points to alive in
    the returned list)."""
    B, H, d = q.shape
    keep = []

    def f(t):
        t = _f32(t)
        keep.append(t)
        return t

    pos = pos.to(torch.int32).contiguous()
    keep.append(pos)
    if out is None and partial_out is None:
        out = torch.empty_like(q)
    HI = dI = 0
    qI_dt = kI_dt = 0
    if qI is not None:
        _, HI, dI = qI.shape
        qI_dt, kI_dt = _dt(qI), _dt(kI)
    # a uint8 cache holds FP8 KV rows (include/csahca.h: e4m3 non-RoPE dims with
    # one fp32 scale per 64, bf16 RoPE dims)
    kv_dt = N.E4M3 if kv_cache.dtype == torch.uint8 else _dt(q)
    args = N.DecodeArgs(kind=N.CSA if kind == "csa" else N.HCA, dtype=_dt(q), B=B, H=H, d=d,
                        N_cap=kv_cache.shape[1], m=m, w=win.shape[1] if win is not None else 0,
                        kv_dtype=kv_dt,
                        rope_dims=rope_dims, rope_base=rope_base, eps=eps, scale=scale,
                        q_norm=int(bool(q_norm)), k=k, HI=HI, dI=dI, qI_dtype=qI_dt,
                        kI_dtype=kI_dt, q=_ptr(q), pos=_ptr(pos), q_gain=_ptr(f(q_gain)),
                        kv_cache=_ptr(kv_cache), win=_ptr(win), sinks=_ptr(f(sinks)),
                        qI=_ptr(qI), wI=_ptr(f(wI)), kI=_ptr(kI), kI_scale=_ptr(f(kI_scale)),
                        idx_in=_ptr(idx_in), idx_out=_ptr(idx_out), out=_ptr(out),
                        entry_base=int(entry_base), partial_out=_ptr(partial_out),
                        skip_window=int(bool(skip_window)))
    return args, out, keep


def compressed_attn_decode(kind, q, pos, kv_cache, win, sinks, *, m, rope_dims, k=0, qI=None,
                           wI=None, kI=None, kI_scale=None, idx_in=None, idx_out=None,
                           q_gain=None, q_norm=True, rope_base=10000.0, eps=1e-6, scale=0.0,
                           out=None, entry_base=0, partial_out=None, skip_window=False,
                           workspace=None, stream=None):
    """One decode step of one CSA or HCA layer for B sequences (one new query
    each at pos[b]); CSA selects with the lightning indexer unless idx_in is
    given.  Returns out [B, H, d], or partial_out [B, 2H + H*d] f32 (this
    rank's share of a context-parallel layer whose cache shard starts at
    global entry entry_base) when that is given."""
    args, out, keep = decode_args(kind, q, pos, kv_cache, win, sinks, m=m, rope_dims=rope_dims,
                                  k=k, qI=qI, wI=wI, kI=kI, kI_scale=kI_scale, idx_in=idx_in,
                                  idx_out=idx_out, q_gain=q_gain, q_norm=q_norm,
                                  rope_base=rope_base, eps=eps, scale=scale, out=out,
                                  entry_base=entry_base, partial_out=partial_out,
                                  skip_window=skip_window)
    L = N.lib()
    ws_bytes = L.csahca_decode_workspace_size(C.byref(args))
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    args.workspace = _ptr(workspace)
    args.workspace_bytes = workspace.numel()
    N.check(L.compressed_attn_decode(C.byref(args), _stream(stream)), "compressed_attn_decode")
    del keep
    return out if partial_out is None else partial_out


def decode_compress_args(kind, pos, streams, ring, kv_cache, *, m, bias_a, bias_b=None, kv_raw=None,
                         win=None, kv_gain=None, kv_norm=True, rope_dims=0, rope_base=10000.0,
                         eps=1e-6, istreams=None, ibias_a=None, ibias_b=None, iring=None, kI=None,
                         kI_scale=None, entry_base=0):
    """Build the DecodeCompressArgs struct (and the list of tensors it points to).

    streams: (a, b, za, zb) for "csa" or (a, za) for "hca", each [B, d];
    ring [B, R, S, d]; istreams: (ia, ib, iza, izb) [B, dI] with iring
    [B, 2m, 4, dI] and kI / kI_scale (csa only, optional)."""
    B, d = streams[0].shape
    keep = []

    def f(t):
        t = _f32(t)
        keep.append(t)
        return t

    pos = pos.to(torch.int32).contiguous()
    keep.append(pos)
    csa = kind == "csa"
    a, b, za, zb = (streams if csa else (streams[0], None, streams[1], None))
    dI = 0
    ia = ib = iza = izb = None
    if csa and istreams is not None:
        ia, ib, iza, izb = istreams
        dI = ia.shape[1]
        if kI is None or iring is None or ibias_a is None or ibias_b is None:
            raise ValueError("decode_compress: indexer streams need iring, ibias_a, ibias_b and kI")
    args = N.DecodeCompressArgs(
        kind=N.CSA if csa else N.HCA, dtype=_dt(a), B=B, d=d, m=m, N_cap=kv_cache.shape[1],
        w=win.shape[1] if win is not None else 0, rope_dims=rope_dims, rope_base=rope_base, eps=eps,
        kv_norm=int(bool(kv_norm)), dI=dI, kI_dtype=_dt(kI) if dI else 0,
        kv_dtype=N.E4M3 if kv_cache.dtype == torch.uint8 else _dt(a), entry_base=int(entry_base),
        pos=_ptr(pos), kv_raw=_ptr(kv_raw), a=_ptr(a), b=_ptr(b), za=_ptr(za), zb=_ptr(zb),
        bias_a=_ptr(f(bias_a)), bias_b=_ptr(f(bias_b)), kv_gain=_ptr(f(kv_gain)), ring=_ptr(ring),
        kv_cache=_ptr(kv_cache), win=_ptr(win), ia=_ptr(ia), ib=_ptr(ib), iza=_ptr(iza), izb=_ptr(izb),
        ibias_a=_ptr(f(ibias_a)), ibias_b=_ptr(f(ibias_b)), iring=_ptr(iring), kI=_ptr(kI),
        kI_scale=_ptr(kI_scale))
    return args, keep


def decode_compress(kind, pos, streams, ring, kv_cache, *, m, bias_a, stream=None, **kw):
    """One decode step of one layer's compressors: the new token's raw streams
    into the ring, its window row (if kv_raw and win are given) and, when the
    token completes a block, the new compressed entry (and indexer key) into
    the caches.  Updates ring, win, kv_cache, iring, kI, kI_scale in place."""
    args, keep = decode_compress_args(kind, pos, streams, ring, kv_cache, m=m, bias_a=bias_a, **kw)
    N.check(N.lib().decode_compress(C.byref(args), _stream(stream)), "decode_compress")
    del keep


def cp_partial_floats(H: int, d: int) -> int:
    """Floats of one row's context-parallel attention share: mx[H], l[H], o[H][d]."""
    return 2 * H + H * d


def cp_topk_merge(cand_idx, cand_scores, bases, rank, *, idx_global=None, idx_local=None, stream=None):
    """Stage 1 of context parallelism: the global top-k from every rank's
    candidates.  cand_idx / cand_scores [R, rows, k] (local rows and their
    scores, as indexer_topk writes idx / sel_scores); bases: the R shards'
    first global entries (host ints).  Returns (idx_global, idx_local), each
    [rows, k] int32 in ascending global order, -1 padded; idx_local holds the
    rows of rank `rank` and -1 for the other ranks' entries."""
    R, rows, k = cand_idx.shape
    dev = cand_idx.device
    if idx_global is None:
        idx_global = torch.empty(rows, k, dtype=torch.int32, device=dev)
    if idx_local is None:
        idx_local = torch.empty(rows, k, dtype=torch.int32, device=dev)
    b = (C.c_int32 * R)(*[int(x) for x in bases])
    args = N.CpTopkMergeArgs(R=R, rows=rows, k=k, rank=int(rank), bases=C.cast(b, C.c_void_p),
                             cand_idx=_ptr(cand_idx), cand_scores=_ptr(cand_scores),
                             idx_global=_ptr(idx_global), idx_local=_ptr(idx_local))
    N.check(N.lib().cp_topk_merge(C.byref(args), _stream(stream)), "cp_topk_merge")
    return idx_global, idx_local


def cp_attn_merge(partials, sinks, pos, *, H, d, rope_dims, dtype=torch.bfloat16, rope_base=10000.0,
                  out=None, stream=None):
    """Stage 2 of context parallelism: the layer output [rows, H, d] from the
    ranks' shares partials [R, rows, 2H + H*d] f32, with the sink and the
    output de-rotation by -pos."""
    R, rows, _ = partials.shape
    if out is None:
        out = torch.empty(rows, H, d, dtype=dtype, device=partials.device)
    keep = _f32(sinks)
    pos = pos.to(torch.int32).contiguous()
    args = N.CpMergeArgs(dtype=_dt(out), R=R, rows=rows, H=H, d=d, rope_dims=rope_dims, rope_base=rope_base,
                         partials=_ptr(partials), sinks=_ptr(keep), pos=_ptr(pos), out=_ptr(out))
    N.check(N.lib().cp_attn_merge(C.byref(args), _stream(stream)), "cp_attn_merge")
    return out


def device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    code = N.i32(0)
    N.check(N.lib().csahca_device_error(_stream(stream), C.byref(code)), "csahca_device_error")
    return int(code.value)


def selftest_bounded_wait(stream=None) -> None:
    """Launch the library's failure-path self-test: a kernel whose bounded
    wait gives up; device_error() on the same stream then reports code 1."""
    N.check(N.lib().csahca_selftest_bounded_wait(_stream(stream)), "csahca_selftest_bounded_wait")


def trace_enable(on: bool = True) -> None:
    """Bracket every library kernel launch with CUDA events (see trace_collect)."""
    N.check(N.lib().csahca_trace_enable(int(bool(on))), "csahca_trace_enable")


def trace_collect() -> dict:
    """Per-kernel {name: (launches, total_ms)} of the launches traced since
    the last collect (synchronises their events)."""
    buf = (N.TraceEntry * 64)()
    n = C.c_int(0)
    N.check(N.lib().csahca_trace_collect(buf, 64, C.byref(n)), "csahca_trace_collect")
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms))
            for i in range(n.value)}
