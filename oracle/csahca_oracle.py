"""Float64 CPU oracle for CSA + HCA compressed attention (forward pass).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or call
this module.  The product path (the CUDA library and its Python binding) never
does, and shares no code, table or helper with it.

Every function is the plain definition of one step of the method, written in
float64 with NumPy; inputs given as fp32 / bf16 / e4m3 are upcast exactly.  No
blocking, fusion or reordering beyond what the definition states.

Sources (web pages on DeepSeek-V4; cited by title and section):

* "Paper Breakdown: DeepSeek-V4", section 4 "Hybrid Attention: CSA + HCA":
  - "CSA ... KV Compression": two streams C^a, C^b with logit streams Z^a, Z^b,
    each compressed block uses 2m entries, a softmax with positional biases
    B^a, B^b, and C^Comp_i = sum S^a_j * C^a_j + sum S^b_j * C^b_j.
  - "DSA on Compressed KV": indexer keys compressed the same way, top-k
    selection by the indexer score I_{t,s}, MQA core attention.
  - "Sliding window KV (uncompressed)".
  - "HCA": single stream, ratio 1/m' (m' >> m), no overlap, no selection.
  - "Additional Techniques": query/KV RMSNorm, partial RoPE on the last 64
    dims, sliding window, a learnable attention-sink logit per head.
* "How DeepSeek-V4 architecture and training work together", section "Two
  compressed views of one history": 1,024 selected entries per query and a
  128-token local window.
* "Inside DeepSeek V4", banner "Two compression regimes" (CSA overlapping
  blocks 4x, HCA non-overlapping blocks 128x) and card "Local window" (128
  recent uncompressed KV entries in every CSA and HCA layer).
* "DeepSeek-V4: Anatomy of an Open-Source Frontier Model", key terms
  "Lightning indexer", "CSA", "HCA".

Readings where the pages are silent (each is a fixed constant of this code):

  R1  stream a pools the current block i, stream b the preceding block i-1.
  R2  entry 0 has no preceding block: its stream-b logits are -inf.
  R3  one joint softmax over all 2m logits per channel (weights sum to 1).
  R4  bias indexed by offset r in the block, per channel: shape [m, c].
  R5  K = V = the same compressed (normed, roped) row (one shared KV head).
  R6  RoPE position of entry i is i*m (first token of its block).
  R7  RoPE on the last r dims of q and kv; the rope dims of the output are
      rotated back by -t (the query position).
  R8  indexer score I_{t,i} = sum_j w_{t,j} * ReLU(qI_{t,j} . kI_i); no norm and
      no RoPE on indexer queries or keys.
  R9  entry i (tokens i*m .. (i+1)*m-1) is visible to query t iff (i+1)*m-1 <= t.
  R10 window of query t = tokens max(0, t-w+1) .. t (its own token included);
      window and compressed entries are not de-duplicated.
  R11 the sink adds e^{z_h} to the softmax denominator only.
  R12 RMSNorm eps = 1e-6, optional gain vector.
  R13 RoPE pairs are interleaved (2j, 2j+1) within the last r dims, with
      angle pos * base^(-2j/r), base 10000.
  R14 softmax scale tau = 1/sqrt(d).
  R15 an incomplete trailing block forms no entry.
  R16 top-k ties: the lower index wins; output sorted ascending, -1 padded.
  R17 e4m3 ("fn" variant: bias 7, no infinities) with one fp32 scale per 128
      contiguous elements of a key row.
  R18 indexer queries stay in their own dtype; only keys are e4m3.
  R20 decode caches hold final rows; the window ring holds final rows, slot
      (p mod w) holding position p.
  R21 the decode compressor stores a new e4m3 indexer key with the same
      per-128 rule as R17, every step in float32: scale = amax / 448 (1 for an
      all-zero block), code = nearest e4m3 of x / scale, ties to even,
      saturating at 448.
  R22 between decode steps a compressor keeps the raw streams of its last
      2m (CSA) or m' (HCA) tokens, token p in ring slot p mod 2m (or p mod m');
      the window row and the compressed rows share one norm gain.
  R23 an FP8 KV cache ("Paper Breakdown: DeepSeek-V4", infrastructure table:
      KV storage FP8 for the non-RoPE dims, BF16 for the RoPE dims) stores the
      first d - r dims of a row as e4m3 with one fp32 scale per 64 of them (the
      R21 rule) and the last r dims as bf16; attention reads the rows it
      stands for.  The window ring stays bf16.

Pins (what checks each function against something other than itself, in
``tests/test_oracle_pins.py`` and ``tests/golden/``):

  e4m3_decode           all 256 codes against torch's float8_e4m3fn cast.
  e4m3_encode           torch's round-to-nearest-even float8_e4m3fn cast on
                        random values and on every midpoint between codes;
                        saturation closed form; decode(encode(v)) = v.
  quantize_kv_rows_fp8  the amax element of each 64-block lands on +-448, an
                        all-zero block has scale 1 and zero codes, the RoPE dims
                        are kept bit for bit, and every element of the
                        dequantised row is within half an e4m3 step of it.
  decode_compress_step  run token by token from position 0, it emits exactly
                        the rows csa_pool / hca_pool + finish_rows give for the
                        whole stream, and the window rows of finish_rows.
  csa_pool              hand-worked fixture; constant streams -> 1 (weights sum
                        to 1); equal logits -> plain mean; one-hot logits copy
                        the named token of the named stream/block; causality.
  hca_pool              equals csa_pool with stream b disabled (one stream, no
                        overlap, m = m') and a hand-worked fixture.
  rms_norm              output RMS 1, scale invariance.
  rope                  closed form of one pair, orthogonality, composition,
                        relative-position property.
  indexer_scores        closed forms (ReLU(x)+ReLU(-x) = |x|; orthogonal q).
  top_k_select          brute force rank counting on tiny inputs.
  attend_query          one key row RoPE_p(y), sink -inf: every head's output is
                        RoPE_{p-t}(y), the expected value written as a complex
                        product per pair (p > t included); shifting the query
                        and every key position by the same delta leaves the
                        output unchanged; the same closed form through
                        decode_attention (one selected entry) and
                        prefill_attention (one-token window).
  sink_attention,
  prefill/decode paths  m=1, all entries selected, no window, no RoPE, sink
                        -inf equals torch's scaled_dot_product_attention;
                        identical-keys sink closed form; perturbation
                        causality; decode equals prefill at the same token.
"""

from __future__ import annotations

import numpy as np

RMS_EPS = 1e-6
ROPE_BASE = 10000.0


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------

def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Decode e4m3 ("fn": 1 sign, 4 exponent bits with bias 7, 3 mantissa
    bits, no infinities, S.1111.111 = NaN) bytes to float64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    f = (c & 0x7).astype(np.float64)
    normal = np.ldexp(1.0 + f / 8.0, e - 7)
    subnormal = np.ldexp(f / 8.0, -6)
    val = sign * np.where(e == 0, subnormal, normal)
    return np.where((e == 15) & (f == 7), np.nan, val)


def e4m3_encode(x) -> np.ndarray:
    """Nearest e4m3 ("fn") code of each finite value: the magnitude code whose
    decoded value is closest to |x|, ties to the code with an even last
    mantissa bit, magnitudes beyond the largest finite one (448) saturating
    to it, and the sign bit of x.  Written as the definition: a search over
    the 127 finite magnitudes."""
    x = np.asarray(x, np.float64)
    mags = np.arange(127, dtype=np.uint8)                   # 0x00 .. 0x7E
    vals = e4m3_decode(mags)
    ax = np.minimum(np.abs(x), 448.0)
    dist = np.abs(ax[..., None] - vals)                     # [..., 127]
    best = dist.min(axis=-1, keepdims=True)
    rank = np.where(dist == best, (mags & 1).astype(np.int64), 9)
    code = mags[np.argmin(rank, axis=-1)]
    return np.where(np.signbit(x), code | np.uint8(0x80), code).astype(np.uint8)


def quantize_e4m3_rows_f32(x, block: int = 128):
    """Per-block e4m3 storage of a key row as the decode compressor writes it
    (reading R21): with every step in float32, scale = amax / 448 over each
    ``block`` contiguous elements (1 where amax is 0) and code =
    e4m3_encode(x / scale).  Returns (codes uint8 [..., d], scales f32
    [..., d/block])."""
    x = np.asarray(x, np.float32)
    d = x.shape[-1]
    xb = x.reshape(*x.shape[:-1], d // block, block)
    amax = np.abs(xb).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    q = (xb / scale[..., None]).astype(np.float32)
    return e4m3_encode(q).reshape(x.shape), scale


def quantize_kv_rows_fp8(rows, r: int, block: int = 64):
    """FP8 storage of KV rows (reading R23): the first d - r ("non-RoPE")
    dims as e4m3 codes with one fp32 scale per ``block`` of them, quantised
    exactly as quantize_e4m3_rows_f32; the last r (RoPE) dims kept as given
    (bf16 in the caches).  Returns (codes uint8 [..., d-r], scales f32
    [..., (d-r)/block], rope [..., r] float64)."""
    rows = np.asarray(rows, np.float64)
    nr = rows.shape[-1] - r
    codes, scales = quantize_e4m3_rows_f32(rows[..., :nr], block)
    return codes, scales, rows[..., nr:].copy()


def dequant_kv_rows_fp8(codes, scales, rope, block: int = 64) -> np.ndarray:
    """The KV rows an FP8 cache stands for: decode(code) * scale on the
    non-RoPE dims, the RoPE dims as stored."""
    return np.concatenate([dequant_e4m3_rows(codes, scales, block), np.asarray(rope, np.float64)], axis=-1)


def dequant_e4m3_rows(codes: np.ndarray, scales: np.ndarray, block: int = 128) -> np.ndarray:
    """Key rows from e4m3 codes [..., d] and fp32 scales [..., d/block]:
    element j of a row is decode(code_j) * scale_{j // block} (reading R17)."""
    x = e4m3_decode(codes)
    s = np.repeat(np.asarray(scales, np.float64), block, axis=-1)
    return x * s


# ----------------------------------------------------------------------------
# compressors  ("Paper Breakdown: DeepSeek-V4", section 4, CSA KV Compression
# and HCA)
# ----------------------------------------------------------------------------

def csa_pool(Ca, Cb, Za, Zb, Ba, Bb, m: int) -> np.ndarray:
    """Overlapped two-stream compression, ratio 1/m, window 2m.

    Ca, Cb, Za, Zb: [n, c] token streams.  Ba, Bb: [m, c] positional biases.
    Entry i (0 <= i < n // m), channel c:
        logits  la_r = Za[i*m + r, c] + Ba[r, c]
                lb_r = Zb[(i-1)*m + r, c] + Bb[r, c]     (-inf for i = 0)
        S = softmax over the 2m logits {la, lb} jointly
        C_i[c] = sum_r Sa_r * Ca[i*m + r, c] + sum_r Sb_r * Cb[(i-1)*m + r, c]
    """
    Ca, Cb, Za, Zb = (np.asarray(x, np.float64) for x in (Ca, Cb, Za, Zb))
    Ba, Bb = np.asarray(Ba, np.float64), np.asarray(Bb, np.float64)
    n, c = Ca.shape
    Nc = n // m
    out = np.zeros((Nc, c), np.float64)
    for i in range(Nc):
        cur = slice(i * m, (i + 1) * m)
        la = Za[cur] + Ba
        va = Ca[cur]
        if i == 0:
            lb = np.full((m, c), -np.inf)
            vb = np.zeros((m, c))
        else:
            prev = slice((i - 1) * m, i * m)
            lb = Zb[prev] + Bb
            vb = Cb[prev]
        logits = np.concatenate([la, lb], axis=0)          # [2m, c]
        mx = logits.max(axis=0)
        e = np.exp(logits - mx)
        S = e / e.sum(axis=0)
        out[i] = (S[:m] * va).sum(axis=0) + (S[m:] * vb).sum(axis=0)
    return out


def hca_pool(C, Z, B, m: int) -> np.ndarray:
    """Non-overlapped single-stream compression, ratio 1/m (m = m').

    Entry i, channel c: C_i[c] = sum_r softmax_r(Z[i*m + r, c] + B[r, c]) * C[i*m + r, c].
    """
    C, Z, B = (np.asarray(x, np.float64) for x in (C, Z, B))
    n, c = C.shape
    Nh = n // m
    out = np.zeros((Nh, c), np.float64)
    for i in range(Nh):
        blk = slice(i * m, (i + 1) * m)
        logits = Z[blk] + B
        e = np.exp(logits - logits.max(axis=0))
        S = e / e.sum(axis=0)
        out[i] = (S * C[blk]).sum(axis=0)
    return out


# ----------------------------------------------------------------------------
# RMSNorm and partial RoPE  ("Paper Breakdown: DeepSeek-V4", section 4,
# Additional Techniques)
# ----------------------------------------------------------------------------

def rms_norm(x, gain=None, eps: float = RMS_EPS) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) over the last axis, times gain (if given)."""
    x = np.asarray(x, np.float64)
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    if gain is not None:
        y = y * np.asarray(gain, np.float64)
    return y


def rope(x, pos, r: int, base: float = ROPE_BASE) -> np.ndarray:
    """Rotate the last r dims of x as r/2 interleaved pairs (2j, 2j+1) by
    angle pos * base^(-2j/r).  pos broadcasts against x.shape[:-1]."""
    x = np.array(x, np.float64, copy=True)
    if r == 0:
        return x
    d = x.shape[-1]
    j = np.arange(r // 2, dtype=np.float64)
    theta = base ** (-2.0 * j / r)                            # [r/2]
    ang = np.asarray(pos, np.float64)[..., None] * theta      # [..., r/2]
    cos, sin = np.cos(ang), np.sin(ang)
    x0 = x[..., d - r + 0::2].copy()
    x1 = x[..., d - r + 1::2].copy()
    x[..., d - r + 0::2] = x0 * cos - x1 * sin
    x[..., d - r + 1::2] = x0 * sin + x1 * cos
    return x


def finish_rows(rows, positions, gain, r: int, base: float = ROPE_BASE,
                normalize: bool = True) -> np.ndarray:
    """RoPE_p(RMSNorm(row) * gain) for each row at its position p.
    With normalize=False the norm is skipped (gain ignored)."""
    y = rms_norm(rows, gain) if normalize else np.asarray(rows, np.float64)
    return rope(y, np.asarray(positions), r, base)


# ----------------------------------------------------------------------------
# one decode step of the compressors  ("Paper Breakdown: DeepSeek-V4",
# section 4, CSA KV Compression, HCA, Sliding window KV)
# ----------------------------------------------------------------------------

def decode_compress_step(kind: str, t: int, new, ring, biases, m: int, *, kv_raw=None,
                         gain=None, r: int = 0, base: float = ROPE_BASE,
                         normalize: bool = True):
    """Fold the token at position t into one sequence's compressor state.

    kind "csa": streams a, b, za, zb; kind "hca": a, za.  ``new`` maps each
    stream name to the token's row [c]; ``ring`` maps it to [R, c] holding
    token p in slot p % R for the R = 2m (csa) or m (hca) tokens before t.
    ``biases`` = (bias_a, bias_b) ([m, c] each; bias_b None for hca).
    Returns (ring', entry, window_row):
      ring'       the ring with the new token in slot t % R (reading R22);
      entry       None unless t completes block i = (t+1)/m - 1, else
                  (i, pooled [c] before finishing, finished [c]) where the
                  pooling is csa_pool / hca_pool over the tokens of block i
                  (and block i-1) and finishing is finish_rows at i*m;
      window_row  finish_rows(kv_raw, t) (None without kv_raw).
    """
    streams = ("a", "b", "za", "zb") if kind == "csa" else ("a", "za")
    R = 2 * m if kind == "csa" else m
    ring = {s: np.array(ring[s], np.float64, copy=True) for s in streams}
    for s in streams:
        ring[s][t % R] = np.asarray(new[s], np.float64)
    entry = None
    if (t + 1) % m == 0:
        i = (t + 1) // m - 1
        first = max(i - 1, 0) * m if kind == "csa" else i * m
        toks = np.arange(first, (i + 1) * m)                  # the blocks entry i pools
        seq = {s: ring[s][toks % R] for s in streams}
        if kind == "csa":
            pooled = csa_pool(seq["a"], seq["b"], seq["za"], seq["zb"], biases[0], biases[1], m)[-1]
        else:
            pooled = hca_pool(seq["a"], seq["za"], biases[0], m)[-1]
        entry = (i, pooled, finish_rows(pooled, i * m, gain, r, base, normalize=normalize))
    win_row = None
    if kv_raw is not None:
        win_row = finish_rows(kv_raw, t, gain, r, base, normalize=normalize)
    return ring, entry, win_row


# ----------------------------------------------------------------------------
# visibility, lightning indexer, top-k  ("Paper Breakdown: DeepSeek-V4",
# section 4, DSA on Compressed KV; "How DeepSeek-V4 architecture and training
# work together", "Two compressed views of one history")
# ----------------------------------------------------------------------------

def n_visible(t: int, m: int) -> int:
    """Number of compressed entries visible to query t (reading R9)."""
    return (t + 1) // m


def indexer_scores(qI_t, w_t, KI) -> np.ndarray:
    """I_{t,i} = sum_j w_{t,j} * max(0, qI_{t,j} . KI_i) for every row i of KI.

    qI_t: [H_I, d_I]; w_t: [H_I]; KI: [N, d_I] -> [N].
    """
    dots = np.asarray(KI, np.float64) @ np.asarray(qI_t, np.float64).T   # [N, H_I]
    return np.maximum(dots, 0.0) @ np.asarray(w_t, np.float64)


def top_k_select(scores, k: int) -> np.ndarray:
    """Indices of the k largest scores (all if fewer), ties to the lower
    index, returned sorted ascending and padded with -1 to length k."""
    scores = np.asarray(scores, np.float64)
    v = scores.shape[0]
    if v <= k:
        sel = np.arange(v)
    else:
        order = np.lexsort((np.arange(v), -scores))
        sel = np.sort(order[:k])
    out = np.full(k, -1, np.int64)
    out[: sel.shape[0]] = sel
    return out


def indexer_topk(qI, w, KI, q_pos, m: int, k: int):
    """Top-k selection for a list of queries of one sequence.

    qI: [nq, H_I, d_I]; w: [nq, H_I]; KI: [N, d_I] (already dequantised);
    q_pos: [nq] absolute positions.  Returns (idx [nq, k], scores list) where
    scores[q] holds I over the visible entries of query q.
    """
    nq = len(q_pos)
    idx = np.full((nq, k), -1, np.int64)
    scores = []
    for qi in range(nq):
        v = min(n_visible(int(q_pos[qi]), m), KI.shape[0])
        s = indexer_scores(qI[qi], w[qi], KI[:v])
        scores.append(s)
        idx[qi] = top_k_select(s, k)
    return idx, scores


# ----------------------------------------------------------------------------
# attention with sink  ("Paper Breakdown: DeepSeek-V4", section 4: MQA core
# attention, sliding window, attention sink)
# ----------------------------------------------------------------------------

def sink_attention(q, rows, sinks, tau: float) -> np.ndarray:
    """o_h = sum_j e^{s_hj} rows_j / (e^{z_h} + sum_j e^{s_hj}),
    s_hj = tau * q_h . rows_j; K = V = rows (reading R5, R11).

    q: [H, d]; rows: [J, d]; sinks: [H] -> [H, d].  J may be 0.
    """
    q = np.asarray(q, np.float64)
    rows = np.asarray(rows, np.float64)
    z = np.asarray(sinks, np.float64)
    H, d = q.shape
    if rows.shape[0] == 0:
        return np.zeros((H, d))
    s = tau * (q @ rows.T)                                # [H, J]
    mx = np.maximum(s.max(axis=1), z)
    e = np.exp(s - mx[:, None])
    den = np.exp(z - mx) + e.sum(axis=1)
    return (e @ rows) / den[:, None]


def window_positions(t: int, w: int) -> np.ndarray:
    """Token positions in the window of query t (reading R10)."""
    return np.arange(max(0, t - w + 1), t + 1)


def attend_query(q_final, key_rows, sinks, t: int, r: int, tau: float,
                 base: float = ROPE_BASE) -> np.ndarray:
    """Sink attention of one (normed, roped) query over key_rows, then the
    rope dims of the output rotated back to position 0 (reading R7)."""
    o = sink_attention(q_final, key_rows, sinks, tau)
    return rope(o, -t, r, base)


def prefill_attention(kind: str, q_raw, kv_comp, kv_win_raw, sinks, *, m: int,
                      w: int, r: int, q_gain=None, kv_gain=None, idx=None,
                      tau=None, base: float = ROPE_BASE, rows=None,
                      q_norm: bool = True, kv_norm: bool = True,
                      q_holds_rows: bool = False) -> np.ndarray:
    """Prefill attention for one sequence.

    kind: "csa" (keys = kv_comp[idx[t]]) or "hca" (keys = every visible entry).
    q_raw: [n, H, d] (or, with q_holds_rows, [len(rows), H, d] holding only the
    queries of ``rows``); kv_comp: [N, d] final compressed rows; kv_win_raw:
    [n, d] per-token rows, finished here at their own positions; idx: [n, k]
    (csa).  Returns o for the query positions in ``rows`` (default all).
    """
    q_raw = np.asarray(q_raw, np.float64)
    _, H, d = q_raw.shape
    n = np.asarray(kv_win_raw).shape[0]
    tau = 1.0 / np.sqrt(d) if tau is None else tau
    kv_comp = np.asarray(kv_comp, np.float64)
    rows = np.arange(n) if rows is None else np.asarray(rows)
    out = np.zeros((len(rows), H, d))
    for oi, t in enumerate(rows):
        t = int(t)
        qt = finish_rows(q_raw[oi if q_holds_rows else t], t, q_gain, r, base, normalize=q_norm)
        if kind == "csa":
            sel = np.asarray(idx[t])
            sel = sel[sel >= 0]
            comp = kv_comp[sel]
        else:
            comp = kv_comp[: min(n_visible(t, m), kv_comp.shape[0])]
        wp = window_positions(t, w)
        win = finish_rows(np.asarray(kv_win_raw, np.float64)[wp], wp, kv_gain, r, base,
                          normalize=kv_norm)
        keys = np.concatenate([comp, win], axis=0)
        out[oi] = attend_query(qt, keys, sinks, t, r, tau, base)
    return out


def decode_attention(kind: str, q_raw, pos: int, kv_cache, win_ring, sinks, *,
                     m: int, w: int, r: int, q_gain=None, sel=None, tau=None,
                     base: float = ROPE_BASE, q_norm: bool = True) -> np.ndarray:
    """One decode step of one sequence for one layer.

    q_raw: [H, d] new query at position pos; kv_cache: [N_cap, d] final rows
    (entry i valid iff visible to pos); win_ring: [w, d] final rows, slot
    p % w holding position p; sel: selected entry indices (csa; -1 ignored).
    """
    q_raw = np.asarray(q_raw, np.float64)
    H, d = q_raw.shape
    tau = 1.0 / np.sqrt(d) if tau is None else tau
    kv_cache = np.asarray(kv_cache, np.float64)
    qt = finish_rows(q_raw, pos, q_gain, r, base, normalize=q_norm)
    if kind == "csa":
        s = np.asarray(sel)
        comp = kv_cache[s[s >= 0]]
    else:
        comp = kv_cache[: min(n_visible(pos, m), kv_cache.shape[0])]
    wp = window_positions(pos, w)
    win = np.asarray(win_ring, np.float64)[wp % w] if w > 0 else np.zeros((0, d))
    keys = np.concatenate([comp, win], axis=0)
    return attend_query(qt, keys, sinks, pos, r, tau, base)
