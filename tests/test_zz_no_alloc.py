"""indexer_topk_noalloc: the allocation-free variant of indexer_topk.

Some callers cannot allocate device memory at the moment they call the
indexer (code that runs inside a fixed, pre-planned memory pool, or a host
thread that must not enter the allocator).  For them the library keeps the
indexer's scratch (score rows and top-k buffers) in one fixed device array
and takes no workspace.  These tests call both entry points through the C ABI
on the same inputs and require identical selections, on two calls in a row
(the shared array keeps the previous call's contents, so the second call also
checks that whatever must start at zero is cleared).

This file is named so that pytest collects it last.
"""

import ctypes as C

import pytest
import torch

from long_context_compressed_overlapped_b200 import build, native as N, synth

DEV = "cuda"


def _args(qI, w, kI, q_pos, m, k, idx, kI_scale=None):
    B, nq, HI, dI = qI.shape
    kdt = N.E4M3 if kI.dtype == torch.uint8 else (N.BF16 if kI.dtype == torch.bfloat16 else N.F32)
    qdt = N.BF16 if qI.dtype == torch.bfloat16 else N.F32
    return N.IndexerArgs(q_dtype=qdt, k_dtype=kdt, B=B, nq=nq, HI=HI, dI=dI, N=kI.shape[1], m=m, k=k,
                         qI=qI.data_ptr(), w=w.data_ptr(), kI=kI.data_ptr(),
                         kI_scale=kI_scale.data_ptr() if kI_scale is not None else None,
                         q_pos=q_pos.data_ptr(), idx=idx.data_ptr())


def _with_workspace(lib, qI, w, kI, q_pos, m, k, kI_scale=None):
    """The existing entry point, with a caller-allocated workspace."""
    idx = torch.full((qI.shape[0], qI.shape[1], k), -7, dtype=torch.int32, device=DEV)
    a = _args(qI, w, kI, q_pos, m, k, idx, kI_scale)
    nbytes = lib.csahca_indexer_workspace_size(C.byref(a))
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=DEV)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    N.check(lib.indexer_topk(C.byref(a), torch.cuda.current_stream().cuda_stream), "indexer_topk")
    torch.cuda.synchronize()
    return idx, nbytes


def _no_alloc(lib, qI, w, kI, q_pos, m, k, kI_scale=None):
    idx = torch.full((qI.shape[0], qI.shape[1], k), -7, dtype=torch.int32, device=DEV)
    a = _args(qI, w, kI, q_pos, m, k, idx, kI_scale)
    N.check(lib.indexer_topk_noalloc(C.byref(a), torch.cuda.current_stream().cuda_stream),
            "indexer_topk_noalloc")
    torch.cuda.synchronize()
    return idx


def _cases():
    """Decode rows long enough for the multi-CTA top-k (bf16 and e4m3 keys,
    ragged key count), and prefill rows that use the single-CTA top-k."""
    D = synth.Draw(31, DEV)
    out = []
    B, ctx = 3, 4 * 40000 + 6
    Nk = ctx // 4
    qI = D.normal("qI_dec", (B, 1, 64, 128), 1.0, torch.bfloat16)
    w = D.normal("w_dec", (B, 1, 64), 1 / 8.0)
    kb = D.normal("kI_dec", (B, Nk, 128), 1.0, torch.bfloat16)
    pos = torch.tensor([[ctx], [ctx - 5], [4 * 1500 + 1]], device=DEV, dtype=torch.int32)
    out.append(("decode bf16 keys", qI, w, kb, pos, None))
    codes, scales = synth.quantize_e4m3_rows(kb)
    out.append(("decode e4m3 keys", qI, w, codes, pos, scales))
    n, Np = 96, 2048 + 3
    qp = D.normal("qI_pre", (1, n, 64, 128), 1.0, torch.bfloat16)
    wp = D.normal("w_pre", (1, n, 64), 1 / 8.0)
    kp = D.normal("kI_pre", (1, Np, 128), 1.0, torch.bfloat16)
    posp = torch.arange(4 * Np - n, 4 * Np, device=DEV, dtype=torch.int32)[None].contiguous()
    out.append(("prefill bf16 keys", qp, wp, kp, posp, None))
    return out


@pytest.fixture(scope="module")
def lib():
    build.build()
    return N.lib()


@pytest.mark.gpu
def test_noalloc_matches_indexer_topk_twice(lib):
    for name, qI, w, kI, pos, scale in _cases():
        want, nbytes = _with_workspace(lib, qI, w, kI, pos, 4, 1024, scale)
        assert 0 < nbytes <= N.NOALLOC_SCRATCH_BYTES, name
        for call in range(2):
            got = _no_alloc(lib, qI, w, kI, pos, 4, 1024, scale)
            # indices are integers: the two entry points must agree exactly
            assert torch.equal(got, want), f"{name}: call {call + 1} differs from indexer_topk"
    code = N.i32(0)
    N.check(lib.csahca_device_error(torch.cuda.current_stream().cuda_stream, C.byref(code)), "device_error")
    assert code.value == 0


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    """A problem whose scratch exceeds the fixed array is refused before any
    launch (host-side check; runs with or without a GPU)."""
    a = N.IndexerArgs(q_dtype=N.BF16, k_dtype=N.BF16, B=64, nq=1, HI=64, dI=128, N=1 << 20, m=4,
                      k=1024, qI=256, w=256, kI=256, q_pos=256, idx=256)
    assert lib.csahca_indexer_workspace_size(C.byref(a)) > N.NOALLOC_SCRATCH_BYTES
    assert lib.indexer_topk_noalloc(C.byref(a), None) == N.ERR_WORKSPACE
    # invalid arguments are reported exactly as by indexer_topk
    a.k = 0
    assert lib.indexer_topk_noalloc(C.byref(a), None) == N.ERR_INVALID_ARG
