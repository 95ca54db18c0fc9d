"""Pins for the float64 oracle: each check compares it with something other than
itself -- a hand-worked example from the pages' equations, a closed form, an
invariant the pages fix, a library routine it must reduce to, or brute force.

Sources: "Paper Breakdown: DeepSeek-V4", section 4 (CSA KV compression, DSA on
compressed KV, sliding window, HCA, Additional Techniques); "How DeepSeek-V4
architecture and training work together", "Two compressed views of one
history"; "Inside DeepSeek V4", "Two compression regimes" and "Local window".
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import csahca_oracle as O


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- e4m3 ----

def check_e4m3_matches_torch(decode):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = decode(codes)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])


def test_e4m3_decode_all_codes():
    check_e4m3_matches_torch(O.e4m3_decode)


def test_e4m3_block_scales():
    rng = np.random.default_rng(0)
    codes = rng.integers(0, 126, size=(3, 256)).astype(np.uint8)  # finite codes
    scales = np.array([[2.0, 0.5], [1.0, 4.0], [0.25, 8.0]])
    x = O.dequant_e4m3_rows(codes, scales)
    base = O.e4m3_decode(codes)
    assert np.array_equal(x[:, :128], base[:, :128] * scales[:, :1])
    assert np.array_equal(x[:, 128:], base[:, 128:] * scales[:, 1:])


def _e4m3_probe_values():
    """float32 values across the e4m3 range: random magnitudes, every finite
    code value, every midpoint between neighbouring codes (the ties), zero
    and values past the subnormal range, with both signs."""
    rng = np.random.default_rng(3)
    mags = O.e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = (mags[:-1] + mags[1:]) / 2
    rand = rng.uniform(0, 1, 4000) * np.exp2(rng.integers(-12, 9, 4000))
    v = np.concatenate([mags, mids, np.clip(rand, 0, 448), [0.0, 2.0 ** -11, 2.0 ** -10, 1e-30]])
    return np.concatenate([v, -v]).astype(np.float32)


def check_e4m3_encode_matches_torch(encode):
    x = _e4m3_probe_values()
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(encode(x.astype(np.float64)), ref)


def test_e4m3_encode_round_to_nearest_even():
    check_e4m3_encode_matches_torch(O.e4m3_encode)


def test_e4m3_encode_saturates_and_round_trips():
    assert list(O.e4m3_encode(np.array([448.0, 449.0, 480.0, 1e6, -500.0]))) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    assert np.array_equal(O.e4m3_encode(O.e4m3_decode(finite)), finite)


def test_quantize_e4m3_rows_f32():
    from long_context_compressed_overlapped_b200 import synth
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((6, 256)) * np.exp2(rng.integers(-6, 6, (6, 1)))).astype(np.float32)
    x[2, 128:] = 0.0                                        # an all-zero block: scale 1, codes 0
    codes, scales = O.quantize_e4m3_rows_f32(x)
    amax = np.abs(x.reshape(6, 2, 128)).max(axis=-1)
    assert np.array_equal(scales, np.where(amax > 0, amax / np.float32(448), 1).astype(np.float32))
    assert scales[2, 1] == 1.0 and not codes[2, 128:].any()
    # the element of largest magnitude lands on +-448 (code 0x7E or 0xFE)
    j = np.abs(x[0, :128]).argmax()
    assert codes[0, j] & 0x7F == 0x7E
    # the same rule as a torch float32 cast (the harness quantiser)
    tc, ts = synth.quantize_e4m3_rows(torch.from_numpy(x))
    assert np.array_equal(codes, tc.numpy()) and np.array_equal(scales, ts.numpy())


def check_kv_fp8(quant, dequant):
    rng = np.random.default_rng(6)
    d, r = 512, 64
    x = torch.from_numpy(rng.standard_normal((5, d)) * np.exp2(rng.integers(-4, 4, (5, 1)))).to(
        torch.bfloat16).to(torch.float64).numpy()
    x[3, 64:128] = 0.0                                      # an all-zero block
    codes, scales, rope = quant(x, r)
    assert codes.shape == (5, d - r) and scales.shape == (5, (d - r) // 64) and rope.shape == (5, r)
    assert np.array_equal(rope, x[:, d - r:])               # RoPE dims bit for bit
    assert scales[3, 1] == 1.0 and not codes[3, 64:128].any()
    blk = np.abs(x[:, :d - r]).reshape(5, -1, 64)
    j = blk.argmax(axis=-1)
    got = codes.reshape(5, -1, 64)[np.arange(5)[:, None], np.arange(blk.shape[1])[None], j]
    nz = blk.max(axis=-1) > 0
    assert ((got[nz] & 0x7F) == 0x7E).all()                 # the amax element maps to +-448
    y = dequant(codes, scales, rope)
    s_ = np.repeat(scales.astype(np.float64), 64, axis=-1)
    v = np.abs(x[:, :d - r]) / s_
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -6)))         # e4m3 binade (subnormals share 2^-6's)
    half_step = np.exp2(e - 4) * s_                         # 3 mantissa bits: half a step is 2^(e-4)
    assert (np.abs(y[:, :d - r] - x[:, :d - r]) <= half_step * (1 + 1e-6)).all()
    assert np.array_equal(y[:, d - r:], x[:, d - r:])


def test_kv_fp8_rows():
    check_kv_fp8(O.quantize_kv_rows_fp8, O.dequant_kv_rows_fp8)


# ----------------------------------------------------------- compressors ----

def check_csa_golden(pool, fx):
    got = pool(np.array(fx["Ca"]), np.array(fx["Cb"]), np.array(fx["Za"]), np.array(fx["Zb"]),
               np.array(fx["Ba"]), np.array(fx["Bb"]), fx["m"])
    np.testing.assert_allclose(got, np.array(fx["expected"]), rtol=1e-14, atol=1e-13)


def test_csa_pool_golden(golden_dir):
    check_csa_golden(O.csa_pool, _load(golden_dir, "csa_pool_tiny.json"))


def test_hca_pool_golden(golden_dir):
    fx = _load(golden_dir, "hca_pool_tiny.json")
    got = O.hca_pool(np.array(fx["C"]), np.array(fx["Z"]), np.array(fx["B"]), fx["m"])
    np.testing.assert_allclose(got, np.array(fx["expected"]), rtol=1e-14, atol=1e-13)


def _streams(rng, n, c, m):
    return dict(Ca=rng.standard_normal((n, c)), Cb=rng.standard_normal((n, c)),
                Za=rng.standard_normal((n, c)), Zb=rng.standard_normal((n, c)),
                Ba=0.1 * rng.standard_normal((m, c)), Bb=0.1 * rng.standard_normal((m, c)))


def test_csa_pool_weights_sum_to_one():
    """The pool weights are a softmax, so they sum to 1 per channel and
    constant streams pool to the constant whatever the logits."""
    rng = np.random.default_rng(1)
    s = _streams(rng, 37, 5, 4)
    s["Ca"] = np.full((37, 5), 3.0)
    s["Cb"] = np.full((37, 5), 3.0)
    out = O.csa_pool(s["Ca"], s["Cb"], s["Za"], s["Zb"], s["Ba"], s["Bb"], 4)
    assert out.shape == (9, 5)                     # tail of 1 token forms no entry
    np.testing.assert_allclose(out, 3.0, rtol=1e-14)


def test_csa_pool_equal_logits_is_mean():
    rng = np.random.default_rng(2)
    n, c, m = 24, 3, 4
    Ca, Cb = rng.standard_normal((n, c)), rng.standard_normal((n, c))
    z, b = np.zeros((n, c)), np.zeros((m, c))
    out = O.csa_pool(Ca, Cb, z, z, b, b, m)
    for i in range(n // m):
        toks = [Ca[i * m + r] for r in range(m)]
        if i > 0:
            toks += [Cb[(i - 1) * m + r] for r in range(m)]
        np.testing.assert_allclose(out[i], sum(toks) / len(toks), rtol=1e-13)


@pytest.mark.parametrize("stream,blk_off,r", [("a", 0, 0), ("a", 0, 3), ("b", -1, 0), ("b", -1, 2)])
def test_csa_pool_one_hot_copies_named_token(stream, blk_off, r):
    """A dominant logit on token (block i + blk_off, offset r) of one stream
    makes entry i copy that token's value: pins which block each stream pools."""
    rng = np.random.default_rng(3)
    n, c, m, i = 32, 4, 4, 5
    s = _streams(rng, n, c, m)
    tok = (i + blk_off) * m + r
    key = "Za" if stream == "a" else "Zb"
    s[key][tok, :] = 60.0
    out = O.csa_pool(s["Ca"], s["Cb"], s["Za"], s["Zb"], s["Ba"], s["Bb"], m)
    val = s["Ca" if stream == "a" else "Cb"][tok]
    np.testing.assert_allclose(out[i], val, rtol=1e-12, atol=1e-12)


def test_csa_pool_dependencies():
    """Entry i depends on stream a of block i and stream b of block i-1 only."""
    rng = np.random.default_rng(4)
    n, c, m = 40, 3, 4
    base = _streams(rng, n, c, m)
    ref = O.csa_pool(*(base[k] for k in ("Ca", "Cb", "Za", "Zb", "Ba", "Bb")), m)
    for key in ("Ca", "Cb", "Za", "Zb"):
        for tok in (0, 7, 13, 22, 39):
            s = {k: v.copy() for k, v in base.items()}
            s[key][tok] += 1.0
            out = O.csa_pool(*(s[k] for k in ("Ca", "Cb", "Za", "Zb", "Ba", "Bb")), m)
            blk = tok // m
            for i in range(n // m):
                dep = (i == blk) if key in ("Ca", "Za") else (i == blk + 1)
                changed = not np.allclose(out[i], ref[i], rtol=0, atol=1e-15)
                assert changed == dep, (key, tok, i)


def test_hca_equals_csa_with_stream_b_disabled():
    """HCA(m') is CSA with m = m', one stream and no overlap ("Paper Breakdown:
    DeepSeek-V4", section 4, HCA)."""
    rng = np.random.default_rng(5)
    n, c, m = 200, 6, 16
    s = _streams(rng, n, c, m)
    zb_off = np.full((n, c), -np.inf)
    csa = O.csa_pool(s["Ca"], s["Cb"], s["Za"], zb_off, s["Ba"], s["Bb"], m)
    hca = O.hca_pool(s["Ca"], s["Za"], s["Ba"], m)
    np.testing.assert_allclose(csa, hca, rtol=1e-14, atol=1e-15)


# ----------------------------------------------------------- norm & rope ----

def test_rms_norm_properties():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((5, 64)) * 3.0
    y = O.rms_norm(x)
    np.testing.assert_allclose(np.sqrt((y * y).mean(-1)), 1.0, rtol=1e-6)
    # scale invariance is exact with eps = 0 and holds to ~eps / mean(x^2) otherwise
    np.testing.assert_allclose(O.rms_norm(7.5 * x, eps=0.0), O.rms_norm(x, eps=0.0), rtol=1e-13)
    np.testing.assert_allclose(O.rms_norm(7.5 * x), y, rtol=1e-6)
    g = rng.standard_normal(64)
    np.testing.assert_allclose(O.rms_norm(x, g), y * g, rtol=1e-14)


def check_rope_golden(rope, fx):
    got = rope(np.array(fx["x"]), fx["pos"], fx["r"])
    np.testing.assert_allclose(got, np.array(fx["expected"]), rtol=1e-13, atol=1e-15)


def test_rope_golden(golden_dir):
    check_rope_golden(O.rope, _load(golden_dir, "rope_pairs.json"))


def test_rope_orthogonal_composition_relative():
    rng = np.random.default_rng(7)
    d, r = 32, 16
    x = rng.standard_normal((4, d))
    y = O.rope(x, 123, r)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    np.testing.assert_allclose(y[:, : d - r], x[:, : d - r])
    np.testing.assert_allclose(O.rope(O.rope(x, 40, r), 83, r), y, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(O.rope(y, -123, r), x, rtol=1e-12, atol=1e-13)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    s1 = O.rope(q, 500, r) @ O.rope(k, 440, r)
    s2 = O.rope(q, 60, r) @ O.rope(k, 0, r)
    assert abs(s1 - s2) < 1e-11


# -------------------------------------------------------- indexer & top-k ----

def test_indexer_relu_per_head():
    """ReLU(x) + ReLU(-x) = |x|: with two heads q and -q and unit weights the
    score is |q . k|; one head with weight 2 gives 2 ReLU(q . k)."""
    rng = np.random.default_rng(8)
    q = rng.standard_normal(16)
    K = rng.standard_normal((50, 16))
    s = O.indexer_scores(np.stack([q, -q]), np.array([1.0, 1.0]), K)
    np.testing.assert_allclose(s, np.abs(K @ q), rtol=1e-13)
    s2 = O.indexer_scores(np.stack([q, -q]), np.array([2.0, 0.0]), K)
    np.testing.assert_allclose(s2, 2 * np.maximum(K @ q, 0), rtol=1e-13)
    Kp = K - np.outer(K @ q, q) / (q @ q)                    # orthogonal to q
    np.testing.assert_allclose(O.indexer_scores(q[None], np.array([1.0]), Kp), 0, atol=1e-12)


def check_topk_bruteforce(select):
    rng = np.random.default_rng(9)
    for trial in range(60):
        v = int(rng.integers(0, 14))
        s = rng.integers(-3, 4, size=v).astype(np.float64)   # many ties
        k = int(rng.integers(1, 16))
        got = select(s, k)
        rank = np.array([sum(1 for j in range(v) if s[j] > s[i] or (s[j] == s[i] and j < i))
                         for i in range(v)], dtype=np.int64)
        want = [i for i in range(v) if rank[i] < k]
        want = want + [-1] * (k - len(want))
        assert list(got) == want, (s, k, got, want)


def test_topk_bruteforce():
    check_topk_bruteforce(O.top_k_select)


# -------------------------------------------------------------- attention ----

def test_sink_attention_golden(golden_dir):
    fx = _load(golden_dir, "sink_attention_tiny.json")
    q = np.array(fx["q"])
    got = O.sink_attention(q, np.array(fx["rows"]), np.array(fx["sinks"]), 1 / math.sqrt(q.shape[1]))
    np.testing.assert_allclose(got, np.array(fx["expected"]), rtol=1e-14)


def test_sink_identical_keys_halves_output():
    """J identical keys x with sink z = tau q.x + ln J: o = x / 2 (sink weight
    equals the total key weight)."""
    rng = np.random.default_rng(10)
    H, d, J = 3, 8, 5
    q = rng.standard_normal((H, d))
    x = rng.standard_normal(d)
    tau = 1 / math.sqrt(d)
    z = tau * (q @ x) + math.log(J)
    o = O.sink_attention(q, np.tile(x, (J, 1)), z, tau)
    np.testing.assert_allclose(o, np.tile(x / 2, (H, 1)), rtol=1e-12)


def _tiny_layer(rng, n=40, H=3, d=16, r=8, m=4, HI=2, dI=8, w=6):
    return dict(
        Ca=rng.standard_normal((n, d)), Cb=rng.standard_normal((n, d)),
        Za=rng.standard_normal((n, d)), Zb=rng.standard_normal((n, d)),
        Ba=0.1 * rng.standard_normal((m, d)), Bb=0.1 * rng.standard_normal((m, d)),
        Ia=rng.standard_normal((n, dI)), Ib=rng.standard_normal((n, dI)),
        IZa=rng.standard_normal((n, dI)), IZb=rng.standard_normal((n, dI)),
        IBa=0.1 * rng.standard_normal((m, dI)), IBb=0.1 * rng.standard_normal((m, dI)),
        kv_win=rng.standard_normal((n, d)), q=rng.standard_normal((n, H, d)),
        qI=rng.standard_normal((n, HI, dI)), w=rng.standard_normal((n, HI)),
        sinks=rng.standard_normal(H), n=n, H=H, d=d, r=r, m=m, w_len=w)


def _run_csa_layer(L, k):
    """Full CSA prefill layer from raw streams: compress -> finish -> indexer
    top-k -> attention."""
    n, m, r = L["n"], L["m"], L["r"]
    comp = O.csa_pool(L["Ca"], L["Cb"], L["Za"], L["Zb"], L["Ba"], L["Bb"], m)
    kv = O.finish_rows(comp, np.arange(comp.shape[0]) * m, None, r)
    KI = O.csa_pool(L["Ia"], L["Ib"], L["IZa"], L["IZb"], L["IBa"], L["IBb"], m)
    idx, _ = O.indexer_topk(L["qI"], L["w"], KI, np.arange(n), m, k)
    o = O.prefill_attention("csa", L["q"], kv, L["kv_win"], L["sinks"], m=m, w=L["w_len"],
                            r=r, idx=idx)
    return o, idx, kv


def test_reduces_to_causal_sdpa():
    """m = 1 with stream b disabled makes every token its own entry; with all
    entries selected, no window, no RoPE, no norms and sink -inf the layer is
    textbook causal softmax attention (torch SDPA in float64)."""
    rng = np.random.default_rng(11)
    n, H, d = 24, 4, 16
    Ca = rng.standard_normal((n, d))
    z = rng.standard_normal((n, d))
    comp = O.csa_pool(Ca, Ca, z, np.full((n, d), -np.inf), np.zeros((1, d)), np.zeros((1, d)), 1)
    np.testing.assert_allclose(comp, Ca, rtol=1e-15)
    q = rng.standard_normal((n, H, d))
    idx = np.full((n, n), -1)
    for t in range(n):
        idx[t, : t + 1] = np.arange(t + 1)
    o = O.prefill_attention("csa", q, comp, np.zeros((n, d)), np.full(H, -np.inf), m=1, w=0,
                            r=0, idx=idx, q_norm=False, kv_norm=False)
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]                  # [1, H, n, d]
    kt = torch.from_numpy(Ca)[None, None].expand(1, H, n, d)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, is_causal=True)
    np.testing.assert_allclose(o, ref[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)
    # the HCA path with m = 1 is the same computation
    o2 = O.prefill_attention("hca", q, comp, np.zeros((n, d)), np.full(H, -np.inf), m=1, w=0,
                             r=0, q_norm=False, kv_norm=False)
    np.testing.assert_allclose(o2, o, rtol=1e-13, atol=1e-14)


def test_window_alone_is_sliding_window_sdpa():
    """No compressed entries visible (m > n) and no sink: the layer is causal
    sliding-window attention over the finished window rows."""
    rng = np.random.default_rng(12)
    n, H, d, w = 20, 2, 8, 5
    q = rng.standard_normal((n, H, d))
    kw = rng.standard_normal((n, d))
    o = O.prefill_attention("hca", q, np.zeros((0, d)), kw, np.full(H, -np.inf), m=64, w=w,
                            r=0, q_norm=False, kv_norm=False)
    mask = torch.zeros(n, n, dtype=torch.bool)
    for t in range(n):
        mask[t, max(0, t - w + 1): t + 1] = True
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(kw)[None, None].expand(1, H, n, d)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, attn_mask=mask)
    np.testing.assert_allclose(o, ref[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)


def test_hca_equals_csa_with_all_entries_selected():
    """At the attention level: dense HCA over the visible entries equals CSA
    whose top-k keeps every visible entry."""
    rng = np.random.default_rng(13)
    n, H, d, m, w, r = 64, 2, 16, 8, 5, 8
    kv = rng.standard_normal((n // m, d))
    q = rng.standard_normal((n, H, d))
    kw = rng.standard_normal((n, d))
    sinks = rng.standard_normal(H)
    idx = np.full((n, n // m), -1)
    for t in range(n):
        v = O.n_visible(t, m)
        idx[t, :v] = np.arange(v)
    a = O.prefill_attention("hca", q, kv, kw, sinks, m=m, w=w, r=r)
    b = O.prefill_attention("csa", q, kv, kw, sinks, m=m, w=w, r=r, idx=idx)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)


def test_causality_by_perturbation():
    """Perturbing every input at tokens > t leaves o_t and Sel_t unchanged."""
    rng = np.random.default_rng(14)
    L = _tiny_layer(rng)
    o, idx, _ = _run_csa_layer(L, k=3)
    t = 22
    L2 = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in L.items()}
    for key in ("Ca", "Cb", "Za", "Zb", "Ia", "Ib", "IZa", "IZb", "kv_win", "q", "qI", "w"):
        L2[key][t + 1:] += rng.standard_normal(L2[key][t + 1:].shape)
    o2, idx2, _ = _run_csa_layer(L2, k=3)
    np.testing.assert_array_equal(idx[: t + 1], idx2[: t + 1])
    np.testing.assert_allclose(o[: t + 1], o2[: t + 1], rtol=0, atol=0)
    assert not np.allclose(o[t + 1:], o2[t + 1:])


def test_visibility_boundary():
    """Entry i becomes visible exactly at t = (i+1)m - 1: perturbing the tokens
    of block i changes o_t for that t and not for t - 1 (dense HCA, so
    visibility alone decides)."""
    rng = np.random.default_rng(15)
    n, H, d, m, w = 48, 2, 8, 8, 3
    C, Z, B = rng.standard_normal((n, d)), rng.standard_normal((n, d)), 0.1 * rng.standard_normal((m, d))
    q, kw, sinks = rng.standard_normal((n, H, d)), rng.standard_normal((n, d)), rng.standard_normal(H)

    def run(C):
        kv = O.finish_rows(O.hca_pool(C, Z, B, m), np.arange(n // m) * m, None, 4)
        return O.prefill_attention("hca", q, kv, kw, sinks, m=m, w=w, r=4)

    ref = run(C)
    for i in range(n // m):
        C2 = C.copy()
        C2[i * m:(i + 1) * m] += 1.0
        out = run(C2)
        t = (i + 1) * m - 1
        assert np.allclose(out[t - 1], ref[t - 1], rtol=0, atol=0)
        assert not np.allclose(out[t], ref[t])


def test_topk_keeps_all_when_few_visible():
    rng = np.random.default_rng(16)
    L = _tiny_layer(rng)
    _, idx, _ = _run_csa_layer(L, k=5)
    for t in range(L["n"]):
        v = O.n_visible(t, L["m"])
        if v <= 5:
            assert list(idx[t]) == list(range(v)) + [-1] * (5 - v)
        else:
            assert (idx[t] >= 0).all() and (np.diff(idx[t]) > 0).all() and idx[t].max() < v


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_decode_equals_prefill(kind):
    """A decode step at position p over caches built from the same tokens
    gives the prefill output at t = p (ring slot p mod w holds position p)."""
    rng = np.random.default_rng(17)
    L = _tiny_layer(rng, n=45, w=7)
    n, m, r, w = L["n"], L["m"], L["r"], L["w_len"]
    if kind == "csa":
        o, idx, kv = _run_csa_layer(L, k=4)
    else:
        kv = O.finish_rows(O.hca_pool(L["Ca"], L["Za"], L["Ba"], m), np.arange(n // m) * m, None, r)
        o = O.prefill_attention("hca", L["q"], kv, L["kv_win"], L["sinks"], m=m, w=w, r=r)
    win_final = O.finish_rows(L["kv_win"], np.arange(n), None, r)
    for p in (n - 1, 30, 3):
        ring = np.zeros((w, L["d"]))
        for s in O.window_positions(p, w):
            ring[s % w] = win_final[s]
        sel = idx[p] if kind == "csa" else None
        od = O.decode_attention(kind, L["q"][p], p, kv, ring, L["sinks"], m=m, w=w, r=r, sel=sel)
        np.testing.assert_allclose(od, o[p], rtol=1e-12, atol=1e-14)


# ------------------------------------------------- output de-rotation ----

def _rotate_complex(y, delta, r, base=O.ROPE_BASE):
    """Rotation of the last r dims by delta * base^(-2j/r), written as the
    complex product (y_2j + i y_2j+1) * e^(i delta theta_j): an independent
    statement of what RoPE does to one pair."""
    y = np.array(y, np.float64, copy=True)
    d = y.shape[-1]
    theta = base ** (-2.0 * np.arange(r // 2) / r)
    z = (y[..., d - r::2] + 1j * y[..., d - r + 1::2]) * np.exp(1j * np.asarray(delta, np.float64)[..., None] * theta)
    y[..., d - r::2] = z.real
    y[..., d - r + 1::2] = z.imag
    return y


def check_output_derotation(attend):
    """Reading R7 ("relative position on core outputs"): the output's rope
    dims are rotated back by -t, so
      (a) one key row RoPE_p(y) with sink -inf gives every head exactly
          RoPE_{p-t}(y), whatever the query (p > t included);
      (b) shifting the query position and every key position by the same
          delta leaves the output unchanged (only relative positions count).
    ``attend`` has attend_query's signature."""
    rng = np.random.default_rng(18)
    H, d, r = 3, 16, 8
    tau = 1 / math.sqrt(d)
    no_sink = np.full(H, -np.inf)
    for p, t in [(12, 20), (0, 7), (36, 20), (100, 3), (5, 5)]:
        y = rng.standard_normal(d)
        q = O.rope(rng.standard_normal((H, d)), t, r)
        o = attend(q, _rotate_complex(y, p, r)[None], no_sink, t, r, tau)
        np.testing.assert_allclose(o, np.tile(_rotate_complex(y, p - t, r), (H, 1)), rtol=1e-12, atol=1e-12)
    ys, x = rng.standard_normal((6, d)), rng.standard_normal((H, d))
    ps, t, sinks = np.array([0, 4, 8, 20, 31, 33]), 33, rng.standard_normal(H)
    ref = attend(O.rope(x, t, r), O.rope(ys, ps, r), sinks, t, r, tau)
    for delta in (1, 57, 1000):
        got = attend(O.rope(x, t + delta, r), O.rope(ys, ps + delta, r), sinks, t + delta, r, tau)
        np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)


def test_output_derotation():
    check_output_derotation(O.attend_query)


def test_output_derotation_through_layers():
    """The same closed form through the decode and prefill paths: one selected
    entry (finished at i*m) as the only key, and a one-token window (the
    query's own row, p = t, so the output is the unrotated normed row)."""
    rng = np.random.default_rng(19)
    H, d, r, m, N = 2, 16, 8, 4, 30
    raw = rng.standard_normal((N, d))
    gain = 1 + 0.1 * rng.standard_normal(d)
    normed = raw / np.sqrt((raw * raw).mean(-1, keepdims=True) + O.RMS_EPS) * gain
    kv = O.finish_rows(raw, np.arange(N) * m, gain, r)
    no_sink = np.full(H, -np.inf)
    for i, pos in [(3, 50), (7, 29), (20, 41)]:
        od = O.decode_attention("csa", rng.standard_normal((H, d)), pos, kv, np.zeros((0, d)), no_sink,
                                m=m, w=0, r=r, sel=np.array([i, -1]))
        np.testing.assert_allclose(od, np.tile(_rotate_complex(normed[i], i * m - pos, r), (H, 1)),
                                   rtol=1e-12, atol=1e-12)
    n = 24
    op = O.prefill_attention("hca", rng.standard_normal((n, H, d)), np.zeros((0, d)), raw[:n], no_sink,
                             m=64, w=1, r=r, kv_gain=gain)
    np.testing.assert_allclose(op, np.repeat(normed[:n, None], H, axis=1), rtol=1e-12, atol=1e-12)


# ------------------------------------------------ decode compressor step ----

def _decode_stream(kind, n, c, m, seed):
    rng = np.random.default_rng(seed)
    names = ("a", "b", "za", "zb") if kind == "csa" else ("a", "za")
    st = {s: rng.standard_normal((n, c)) for s in names}
    biases = (0.1 * rng.standard_normal((m, c)), 0.1 * rng.standard_normal((m, c)) if kind == "csa" else None)
    return st, biases, rng.standard_normal((n, c)), rng


def check_decode_compress_step(step, kind):
    n, c, r = 40, 16, 4
    m = 4 if kind == "csa" else 8
    R = 2 * m if kind == "csa" else m
    st, biases, kv_raw, rng = _decode_stream(kind, n, c, m, 7 if kind == "csa" else 8)
    gain = 1 + 0.1 * rng.standard_normal(c)
    ring = {s: rng.standard_normal((R, c)) * 1e3 for s in st}    # garbage before position 0
    if kind == "csa":
        pooled = O.csa_pool(st["a"], st["b"], st["za"], st["zb"], biases[0], biases[1], m)
    else:
        pooled = O.hca_pool(st["a"], st["za"], biases[0], m)
    want = O.finish_rows(pooled, np.arange(pooled.shape[0]) * m, gain, r)
    emitted = []
    for t in range(n):
        ring, entry, win = step(kind, t, {s: st[s][t] for s in st}, ring, biases, m,
                                kv_raw=kv_raw[t], gain=gain, r=r)
        np.testing.assert_allclose(win, O.finish_rows(kv_raw[t], t, gain, r), rtol=1e-13, atol=1e-13)
        assert (entry is not None) == ((t + 1) % m == 0)
        if entry is not None:
            i, raw, fin = entry
            assert i == (t + 1) // m - 1
            np.testing.assert_allclose(raw, pooled[i], rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(fin, want[i], rtol=1e-13, atol=1e-13)
            emitted.append(i)
    assert emitted == list(range(n // m))


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_decode_compress_step_equals_whole_stream(kind):
    check_decode_compress_step(O.decode_compress_step, kind)


# --------------------------------------------- planted mistakes are caught ----

def test_pins_catch_planted_mistakes(golden_dir):
    """Plant plausible mistakes in copies of oracle functions and check that
    a pin fails for each (the pins are not vacuous)."""
    fx = _load(golden_dir, "csa_pool_tiny.json")

    def pool_wrong_block(Ca, Cb, Za, Zb, Ba, Bb, m):      # stream b on block i, not i-1
        Cb2 = np.roll(np.asarray(Cb, float), -m, axis=0)
        Zb2 = np.roll(np.asarray(Zb, float), -m, axis=0)
        return O.csa_pool(Ca, Cb2, Za, Zb2, Ba, Bb, m)

    def pool_dropped_b(Ca, Cb, Za, Zb, Ba, Bb, m):         # stream b term dropped
        return O.csa_pool(Ca, np.zeros_like(np.asarray(Cb, float)), Za, Zb, Ba, Bb, m)

    for bad in (pool_wrong_block, pool_dropped_b):
        with pytest.raises(AssertionError):
            check_csa_golden(bad, fx)

    rfx = _load(golden_dir, "rope_pairs.json")

    def rope_wrong_sign(x, pos, r, base=O.ROPE_BASE):
        return O.rope(x, -np.asarray(pos), r, base)

    def rope_half_split(x, pos, r, base=O.ROPE_BASE):      # rotate-half pairing
        x = np.asarray(x, float)
        d = x.shape[-1]
        perm = np.arange(d)
        perm[d - r:] = np.concatenate([np.arange(d - r, d, 2), np.arange(d - r + 1, d, 2)])
        y = O.rope(x[..., perm], pos, r, base)
        out = np.empty_like(y)
        out[..., perm] = y
        return out

    for bad in (rope_wrong_sign, rope_half_split):
        with pytest.raises(AssertionError):
            check_rope_golden(bad, rfx)

    def topk_ties_high(scores, k):                          # ties to the higher index
        s = np.asarray(scores, float)
        v = s.shape[0]
        if v <= k:
            sel = np.arange(v)
        else:
            sel = np.sort(np.lexsort((-np.arange(v), -s))[:k])
        out = np.full(k, -1)
        out[: len(sel)] = sel
        return out

    with pytest.raises(AssertionError):
        check_topk_bruteforce(topk_ties_high)

    def decode_bias_wrong(codes):                           # exponent bias 8
        return O.e4m3_decode(codes) / 2

    with pytest.raises(AssertionError):
        check_e4m3_matches_torch(decode_bias_wrong)

    def encode_ties_away(x):                                # ties away from zero
        x = np.asarray(x, float)
        c = O.e4m3_encode(x)
        up = (c & 0x7F) < 0x7E
        nxt = O.e4m3_decode(np.where(up, c + 1, c).astype(np.uint8))
        tie = up & (np.abs(np.abs(nxt) - np.abs(x)) == np.abs(np.abs(x) - np.abs(O.e4m3_decode(c))))
        return np.where(tie & (np.abs(x) > np.abs(O.e4m3_decode(c))), c + 1, c).astype(np.uint8)

    with pytest.raises(AssertionError):
        check_e4m3_encode_matches_torch(encode_ties_away)

    def step_ring_not_kept(kind, t, new, ring, biases, m, **kw):      # new token never stored
        _, entry, win = O.decode_compress_step(kind, t, new, ring, biases, m, **kw)
        return ring, entry, win

    def step_rope_at_last_token(kind, t, new, ring, biases, m, *, gain=None, r=0, **kw):
        out_ring, entry, win = O.decode_compress_step(kind, t, new, ring, biases, m, gain=gain, r=r, **kw)
        if entry is not None:
            i, raw, _ = entry
            entry = (i, raw, O.finish_rows(raw, t, gain, r))
        return out_ring, entry, win

    def kv_quant_block_128(rows, r, block=64):              # scales per 128, read per 64
        return O.quantize_kv_rows_fp8(rows, r, 128)

    def kv_quant_rope_quantised(rows, r, block=64):         # RoPE dims through e4m3 too
        c, s, rope = O.quantize_kv_rows_fp8(rows, r, block)
        return c, s, O.e4m3_decode(O.e4m3_encode(rope)).astype(np.float64)

    for bad in (kv_quant_block_128, kv_quant_rope_quantised):
        with pytest.raises((AssertionError, ValueError)):
            check_kv_fp8(bad, O.dequant_kv_rows_fp8)

    for kind in ("csa", "hca"):
        for bad in (step_ring_not_kept, step_rope_at_last_token):
            with pytest.raises(AssertionError):
                check_decode_compress_step(bad, kind)

    def attend_rotated_forward(q, rows, sinks, t, r, tau, base=O.ROPE_BASE):     # +t, not -t
        return O.rope(O.sink_attention(q, rows, sinks, tau), t, r, base)

    def attend_not_rotated(q, rows, sinks, t, r, tau, base=O.ROPE_BASE):         # no de-rotation
        return O.sink_attention(q, rows, sinks, tau)

    for bad in (attend_rotated_forward, attend_not_rotated):
        with pytest.raises(AssertionError):
            check_output_derotation(bad)
