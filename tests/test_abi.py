"""The C-ABI library loads on a machine without a GPU, exports every symbol
include/csahca.h declares, its structs match the ctypes mirrors, and host-side
validation rejects bad arguments before any launch (no compute is run)."""

import ctypes as C
import os
import re

import pytest

from long_context_compressed_overlapped_b200 import build, native as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    build.build()
    return N.lib()


def declared_functions():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", src,
                             flags=re.M):
            names.add(m.group(1))
    names.discard("if")
    return sorted(names)


def test_header_declares_the_five_calls():
    names = declared_functions()
    for f in ("csa_compress", "hca_compress", "indexer_topk", "compressed_attn_prefill",
              "compressed_attn_decode"):
        assert f in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 12
    for name in names:
        assert hasattr(lib, name), f"libcsahca.so does not export {name}"
        assert name in N.SIGNATURES, f"binding has no signature for {name}"


def test_struct_sizes_match(lib):
    for which, st in N.STRUCTS.items():
        assert lib.csahca_struct_size(which) == C.sizeof(st)
    assert lib.csahca_struct_size(99) == -1
    assert lib.csahca_abi_version() == N.ABI_VERSION == 4


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert lib.csahca_status_string(code).decode() not in ("", "unknown status")


def test_validation_rejects_before_launch(lib):
    assert lib.csa_compress(None, None) == N.ERR_INVALID_ARG
    a = N.CompressArgs(dtype=N.BF16, B=1, n=64, c=20, m=4)        # c % 8 != 0 for bf16
    assert lib.csa_compress(C.byref(a), None) == N.ERR_UNSUPPORTED
    a = N.CompressArgs(dtype=7, B=1, n=64, c=64, m=4)
    assert lib.csa_compress(C.byref(a), None) == N.ERR_INVALID_ARG
    a = N.CompressArgs(dtype=N.F32, B=1, n=64, c=64, m=4, rope_dims=3)
    assert lib.hca_compress(C.byref(a), None) == N.ERR_INVALID_ARG
    a = N.CompressArgs(dtype=N.F32, B=1, n=64, c=64, m=4, num_blocks=-1, a=8, za=16, bias_a=32, out=48)
    assert lib.hca_compress(C.byref(a), None) == N.ERR_ALIGNMENT
    # empty work is a no-op that needs no device
    a = N.CompressArgs(dtype=N.F32, B=0, n=64, c=64, m=4)
    assert lib.csa_compress(C.byref(a), None) == N.OK
    ia = N.IndexerArgs(q_dtype=N.BF16, k_dtype=N.F32, B=1, nq=1, HI=2, dI=32, N=8, m=4, k=4)
    assert lib.indexer_topk(C.byref(ia), None) == N.ERR_UNSUPPORTED   # mixed q/k dtypes
    ia = N.IndexerArgs(q_dtype=N.BF16, k_dtype=N.E4M3, B=1, nq=1, HI=2, dI=64, N=8, m=4, k=4)
    assert lib.indexer_topk(C.byref(ia), None) == N.ERR_UNSUPPORTED   # e4m3 needs dI % 128
    ia = N.IndexerArgs(q_dtype=N.F32, k_dtype=N.F32, B=1, nq=1, HI=2, dI=32, N=8, m=4, k=0)
    assert lib.indexer_topk(C.byref(ia), None) == N.ERR_INVALID_ARG
    aa = N.AttnArgs(kind=5, dtype=N.F32, B=1, n=4, H=1, d=64, m=4)
    assert lib.compressed_attn_prefill(C.byref(aa), None) == N.ERR_INVALID_ARG
    aa = N.AttnArgs(kind=N.CSA, dtype=N.F32, B=1, n=4, H=1, d=64, m=4, k=4, w=2,
                    q=16, sinks=16, out=16, kv_win=16)                 # CSA without idx
    assert lib.compressed_attn_prefill(C.byref(aa), None) == N.ERR_INVALID_ARG
    da = N.DecodeArgs(kind=N.HCA, dtype=N.BF16, B=1, H=4, d=48, N_cap=4, m=4)
    assert lib.compressed_attn_decode(C.byref(da), None) == N.ERR_UNSUPPORTED
    assert lib.decode_compress(None, None) == N.ERR_INVALID_ARG
    dc = N.DecodeCompressArgs(kind=N.HCA, dtype=N.BF16, B=1, d=96, m=128, N_cap=4)  # d % 64 != 0
    assert lib.decode_compress(C.byref(dc), None) == N.ERR_UNSUPPORTED
    dc = N.DecodeCompressArgs(kind=N.CSA, dtype=N.F32, B=1, d=64, m=4, N_cap=4, dI=128, kI_dtype=N.E4M3)
    assert lib.decode_compress(C.byref(dc), None) == N.ERR_UNSUPPORTED   # e4m3 keys need bf16 rows
    dc = N.DecodeCompressArgs(kind=N.CSA, dtype=N.BF16, B=1, d=512, m=4, N_cap=4, dI=192, kI_dtype=N.BF16)
    assert lib.decode_compress(C.byref(dc), None) == N.ERR_UNSUPPORTED   # dI / 8 must divide 128
    dc = N.DecodeCompressArgs(kind=N.CSA, dtype=N.BF16, B=1, d=512, m=4, N_cap=4, rope_dims=3)
    assert lib.decode_compress(C.byref(dc), None) == N.ERR_INVALID_ARG
    dc = N.DecodeCompressArgs(kind=N.CSA, dtype=N.BF16, B=1, d=512, m=4, N_cap=4, rope_dims=130)
    assert lib.decode_compress(C.byref(dc), None) == N.ERR_UNSUPPORTED   # at most 64 RoPE pairs
    dc = N.DecodeCompressArgs(kind=N.HCA, dtype=N.BF16, B=1, d=512, m=128, N_cap=4, pos=16, a=16, za=16,
                              bias_a=16, ring=16, kv_cache=16)        # HCA needs no b / zb
    dc.kv_cache = 24
    assert lib.decode_compress(C.byref(dc), None) == N.ERR_ALIGNMENT
    dc = N.DecodeCompressArgs(kind=N.CSA, dtype=N.BF16, B=0, d=512, m=4, N_cap=4)
    assert lib.decode_compress(C.byref(dc), None) == N.OK                 # empty batch: no-op
    dc = N.DecodeCompressArgs(kind=N.CSA, dtype=N.BF16, B=1, d=512, m=4, N_cap=4, entry_base=-1)
    assert lib.decode_compress(C.byref(dc), None) == N.ERR_INVALID_ARG


def test_context_parallel_validation(lib):
    """The context-parallel arguments are checked on the host: shard offsets,
    rank counts, the tensor-core-only shapes and a CSA shard's selection."""
    ia = N.IndexerArgs(q_dtype=N.F32, k_dtype=N.F32, B=1, nq=1, HI=2, dI=32, N=8, m=4, k=4, entry_base=-3)
    assert lib.indexer_topk(C.byref(ia), None) == N.ERR_INVALID_ARG
    ia = N.IndexerArgs(q_dtype=N.F32, k_dtype=N.F32, B=1, nq=1, HI=2, dI=32, N=8, m=4, k=4, qI=16, w=16,
                       kI=16, q_pos=16, idx=16, sel_scores=40)
    assert lib.indexer_topk(C.byref(ia), None) == N.ERR_ALIGNMENT
    # shard arguments on the SIMT shapes (d = 128): not covered
    da = N.DecodeArgs(kind=N.HCA, dtype=N.BF16, B=2, H=4, d=128, N_cap=1000, m=128, w=16, entry_base=1000)
    assert lib.compressed_attn_decode(C.byref(da), None) == N.ERR_UNSUPPORTED
    da = N.DecodeArgs(kind=N.HCA, dtype=N.BF16, B=2, H=4, d=128, N_cap=1000, m=128, w=16, skip_window=1)
    assert lib.compressed_attn_decode(C.byref(da), None) == N.ERR_UNSUPPORTED
    # the tensor-core shapes: a CSA shard past the first needs idx_in
    da = N.DecodeArgs(kind=N.CSA, dtype=N.BF16, B=4, H=64, d=512, N_cap=4096, m=4, w=128, rope_dims=64, k=1024,
                      HI=64, dI=128, qI_dtype=N.BF16, kI_dtype=N.BF16, entry_base=4096)
    assert lib.compressed_attn_decode(C.byref(da), None) == N.ERR_INVALID_ARG
    da.idx_in = 16
    assert lib.csahca_decode_workspace_size(C.byref(da)) > 0
    da.entry_base = -1
    assert lib.compressed_attn_decode(C.byref(da), None) == N.ERR_INVALID_ARG
    bases = (C.c_int32 * 2)(0, 100)
    tm = N.CpTopkMergeArgs(R=2, rows=1, k=8, rank=0, bases=C.cast(bases, C.c_void_p), cand_idx=16,
                           cand_scores=16, idx_local=16)
    tm.rank = 2
    assert lib.cp_topk_merge(C.byref(tm), None) == N.ERR_INVALID_ARG       # rank outside 0 .. R-1
    tm.rank, tm.R = 0, 65
    assert lib.cp_topk_merge(C.byref(tm), None) == N.ERR_UNSUPPORTED       # more ranks than CP_MAX_RANKS
    tm.R, tm.k = 8, 4096
    assert lib.cp_topk_merge(C.byref(tm), None) == N.ERR_UNSUPPORTED       # R * k above 16384
    tm.R, tm.k, tm.idx_local = 2, 8, None
    assert lib.cp_topk_merge(C.byref(tm), None) == N.ERR_INVALID_ARG       # no output at all
    tm.idx_local = 16
    neg = (C.c_int32 * 2)(0, -5)
    tm.bases = C.cast(neg, C.c_void_p)
    assert lib.cp_topk_merge(C.byref(tm), None) == N.ERR_INVALID_ARG       # negative shard offset
    tm.rows = 0
    assert lib.cp_topk_merge(C.byref(tm), None) == N.OK                    # no rows: no-op
    mg = N.CpMergeArgs(dtype=N.BF16, R=2, rows=4, H=64, d=512, rope_dims=3, partials=16, sinks=16, pos=16,
                       out=16)
    assert lib.cp_attn_merge(C.byref(mg), None) == N.ERR_INVALID_ARG       # odd RoPE dims
    mg.rope_dims, mg.d = 64, 514
    assert lib.cp_attn_merge(C.byref(mg), None) == N.ERR_UNSUPPORTED       # d % 4 != 0
    mg.d, mg.R = 512, 0
    assert lib.cp_attn_merge(C.byref(mg), None) == N.ERR_INVALID_ARG
    mg.R, mg.out = 2, 24
    assert lib.cp_attn_merge(C.byref(mg), None) == N.ERR_ALIGNMENT


def test_workspace_queries(lib):
    ia = N.IndexerArgs(q_dtype=N.F32, k_dtype=N.F32, B=2, nq=10, HI=2, dI=32, N=100, m=4, k=4)
    assert lib.csahca_indexer_workspace_size(C.byref(ia)) >= 2 * 10 * 100 * 4
    aa = N.AttnArgs(kind=N.HCA, dtype=N.BF16, B=2, n=64, H=4, d=128, m=16, w=8)
    assert lib.csahca_prefill_workspace_size(C.byref(aa)) >= 2 * 64 * 128 * 2
    aa.w = 0
    assert lib.csahca_prefill_workspace_size(C.byref(aa)) == 0
    da = N.DecodeArgs(kind=N.HCA, dtype=N.BF16, B=2, H=4, d=128, N_cap=1000, m=128, w=16)
    assert lib.csahca_decode_workspace_size(C.byref(da)) > 0


def test_no_device_is_reported_not_faked(lib):
    """On a machine without a GPU a valid call must fail with NO_DEVICE:
    there is no CPU path behind the ABI."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    a = N.CompressArgs(dtype=N.F32, B=1, n=64, c=64, m=4, num_blocks=-1, a=16, b=16, za=16, zb=16, bias_a=16,
                       bias_b=16, out=16)
    assert lib.csa_compress(C.byref(a), None) == N.ERR_NO_DEVICE
    dc = N.DecodeCompressArgs(kind=N.HCA, dtype=N.BF16, B=1, d=512, m=128, N_cap=4, pos=16, a=16, za=16,
                              bias_a=16, ring=16, kv_cache=16)
    assert lib.decode_compress(C.byref(dc), None) == N.ERR_NO_DEVICE
    assert lib.csahca_selftest_bounded_wait(None) == N.ERR_NO_DEVICE


def test_kv_row_bytes_matches_the_binding(lib):
    """csahca_kv_row_bytes (the library) against the harness's layout."""
    from long_context_compressed_overlapped_b200 import synth
    assert lib.csahca_kv_row_bytes(N.E4M3, 512, 64) == synth.kv_fp8_row_bytes(512, 64) == 640
    assert lib.csahca_kv_row_bytes(N.E4M3, 512, 128) == synth.kv_fp8_row_bytes(512, 128) == 768
    assert lib.csahca_kv_row_bytes(N.BF16, 512, 64) == 1024
    assert lib.csahca_kv_row_bytes(N.F32, 128, 0) == 512
    assert lib.csahca_kv_row_bytes(N.E4M3, 512, 32) == 0          # RoPE dims not a multiple of 64
