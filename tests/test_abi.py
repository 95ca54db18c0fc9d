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
    assert lib.csahca_abi_version() == 2


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
