"""The algorithmic bytes bench.py divides by, worked out by hand for the
decode_1m step (B = 4, context 1,048,576, CSA / HCA / CSA / HCA, e4m3
indexer keys with one fp32 scale per 128, top-k 1,024, window 128, 64 heads
of 512 bf16 dims)."""

import bench
from long_context_compressed_overlapped_b200 import synth


def test_decode_1m_step_bytes():
    wl = synth.WORKLOADS["decode_1m"]
    ctx = wl.ctx
    # per sequence, CSA layer: 262,144 visible keys of 128 e4m3 bytes + 4 scale bytes,
    # plus the indexer query (64 x 128 bf16) and head weights (64 fp32)
    indexer = 262144 * 132 + 64 * 128 * 2 + 64 * 4
    # attention: 1,024 selected + 128 window rows of 1 KB, plus q and o (64 x 512 bf16 each)
    attn_csa = (1024 + 128) * 1024 + 2 * 64 * 512 * 2
    # HCA: 8,192 visible rows + 128 window rows, plus q and o
    attn_hca = (8192 + 128) * 1024 + 2 * 64 * 512 * 2
    # compressor step at position 1,048,576 (completes no block): the token's streams
    # read and stored in the ring, the raw window row read and the finished row written
    comp_csa = 2 * 4 * 512 * 2 + 2 * 512 * 2 + 2 * 4 * 128 * 2
    comp_hca = 2 * 2 * 512 * 2 + 2 * 512 * 2
    per = bench.decode_bytes_per_kernel(wl, ctx)
    assert per["indexer_scores"] == 4 * indexer
    assert per["attn_decode_csa"] == 4 * attn_csa
    assert per["attn_decode_hca"] == 4 * attn_hca
    assert bench.decode_compress_bytes(wl, "csa", ctx) == 4 * comp_csa
    assert bench.decode_compress_bytes(wl, "hca", ctx) == 4 * comp_hca
    step = 4 * 2 * (indexer + attn_csa + comp_csa + attn_hca + comp_hca)
    assert step == 356_796_416
    assert bench.decode_step_bytes(wl, ctx) == step


def test_compressor_bytes_when_a_block_completes():
    wl = synth.WORKLOADS["decode_1m"]
    t = (1 << 20) - 1                          # completes CSA block 262,143 and HCA block 8,191
    base_csa = 2 * 4 * 512 * 2 + 2 * 512 * 2 + 2 * 4 * 128 * 2
    # the other 7 tokens of blocks i-1, i: value and logit rows; the entry; the e4m3 key + scale
    emit_csa = 7 * 2 * 512 * 2 + 512 * 2 + 7 * 2 * 128 * 2 + 128 + 4
    assert bench.decode_compress_bytes(wl, "csa", t) == 4 * (base_csa + emit_csa)
    base_hca = 2 * 2 * 512 * 2 + 2 * 512 * 2
    emit_hca = 127 * 2 * 512 * 2 + 512 * 2
    assert bench.decode_compress_bytes(wl, "hca", t) == 4 * (base_hca + emit_hca)
    # the first CSA block has no preceding block: 3 other tokens, stream a only
    assert bench.decode_compress_bytes(wl, "csa", 3) == 4 * (base_csa + 3 * 2 * 512 * 2 + 512 * 2 +
                                                             3 * 2 * 128 * 2 + 128 + 4)


def test_prefill_128k_flops_closed_form():
    """csa_prefill_128k: n = 131,072 = 4Q tokens (Q = 32,768), m = 4, k = 1,024,
    w = 128, 64 indexer heads of 128 dims, 64 heads of 512 dims.
    Indexer pairs: sum over u = 1..4Q of floor(u/4) = 2Q^2 - Q.
    Attention keys: selected min(floor(u/4), 1024) -- 2*1024^2 - 2*1024 up to
    u = 4,095, then 1,024 for each of the other 126,977 tokens -- plus the
    window min(128, u): 128*129/2 + (131,072 - 128) * 128."""
    pw = synth.WORKLOADS["csa_prefill_128k"]
    Q = 32768
    pairs = 2 * Q * Q - Q
    keys = (2 * 1024 * 1024 - 2 * 1024) + (131072 - 4096 + 1) * 1024 + 128 * 129 // 2 + (131072 - 128) * 128
    idx_fl, att_fl = bench.prefill_flops(pw)
    assert idx_fl == pairs * 64 * 128 * 2 == 35_183_835_217_920
    assert att_fl == keys * 64 * 512 * 4
    assert keys == 148_888_640
    assert idx_fl + att_fl == 54_698_967_040_000
