"""The harness's FP8 KV row packing (synth.pack_kv_rows_fp8, the library's
row layout in include/csahca.h) against the oracle's FP8 KV quantiser
(reading R23: e4m3 non-RoPE dims with one fp32 scale per 64, the RoPE dims
kept; "Paper Breakdown: DeepSeek-V4", infrastructure table)."""

import numpy as np
import torch

from long_context_compressed_overlapped_b200 import synth
from oracle import csahca_oracle as O


def test_pack_kv_rows_fp8_matches_oracle_quantiser():
    g = torch.Generator().manual_seed(5)
    d, r = 512, 64
    x = (torch.randn(7, d, generator=g) * torch.exp2(torch.randint(-5, 5, (7, 1), generator=g).float()))
    x = x.to(torch.bfloat16)
    x[2, 64:128] = 0                                     # an all-zero block
    packed = synth.pack_kv_rows_fp8(x, r)
    assert packed.dtype == torch.uint8 and packed.shape == (7, synth.kv_fp8_row_bytes(d, r)) == (7, 640)
    codes, scales, rope = synth.unpack_kv_rows_fp8(packed, d, r)
    oc, osc, orope = O.quantize_kv_rows_fp8(x.to(torch.float64).numpy(), r)
    assert np.array_equal(codes.numpy(), oc)
    assert np.array_equal(scales.numpy(), osc)
    assert np.array_equal(rope.to(torch.float64).numpy(), orope)
    assert not packed[:, 604:].any()                     # padding
    rows = O.dequant_kv_rows_fp8(codes.numpy(), scales.numpy(), rope.to(torch.float64).numpy())
    np.testing.assert_array_equal(rows, O.dequant_kv_rows_fp8(oc, osc, orope))


def test_kv_fp8_row_bytes_layout():
    """448 codes + 64 x 2 RoPE bytes + 7 x 4 scale bytes = 604 -> 640; with
    r = 128: 384 + 256 + 24 = 664 -> 768."""
    assert synth.kv_fp8_row_bytes(512, 64) == 640
    assert synth.kv_fp8_row_bytes(512, 128) == 768
