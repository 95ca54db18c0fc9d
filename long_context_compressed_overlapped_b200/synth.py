"""Seeded synthetic inputs for the CSA / HCA attention path.

This module only draws random tensors and changes their storage format (fp32
draw -> round-to-nearest-even to the storage dtype; e4m3 quantisation of
indexer keys with one fp32 scale per 128 elements).  It holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle take their inputs
from here.

Workloads (shapes of the pages' 4x / 128x compression, top-k 1024 and 128-token
window; see "How DeepSeek-V4 architecture and training work together", "Two
compressed views of one history", and "Inside DeepSeek V4", "Two compression
regimes"):

  tiny_csa_f32      B=1 n=512 H=4 d=64 r=16 m=4 H_I=2 d_I=32 k=16 w=16, fp32
  hca_8k_bf16       B=2 n=8192 H=16 d=128 r=64 m'=128 w=128, bf16
  csa_prefill_128k  B=1 n=131072 H=64 d=512 r=64 m=4 H_I=64 d_I=128 k=1024 w=128
  decode_256k       B=8 ctx=262144, one CSA + one HCA layer, bf16 indexer keys
  decode_1m         B=4 ctx=1048576, CSA,HCA,CSA,HCA, e4m3 indexer keys
  decode_1m_fp8kv   decode_1m with FP8 KV cache rows (e4m3 non-RoPE dims with
                    one fp32 scale per 64, bf16 RoPE dims; "Paper Breakdown:
                    DeepSeek-V4", infrastructure table)
"""

from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "f32" or "bf16": storage dtype of activations / caches
    B: int
    H: int
    d: int
    r: int
    w: int
    seed: int
    n: int = 0            # prefill tokens
    m: int = 4            # CSA ratio
    m_hca: int = 128      # HCA ratio
    HI: int = 0
    dI: int = 0
    k: int = 0
    ctx: int = 0          # decode: cached context length (new token at position ctx)
    layers: tuple = ()    # decode layer schedule, e.g. ("csa", "hca")
    kind: str = "csa"     # prefill layer kind
    fp8_keys: bool = False
    fp8_kv: bool = False  # decode caches as FP8 KV rows

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    "tiny_csa_f32": Workload("tiny_csa_f32", "f32", B=1, n=512, H=4, d=64, r=16, m=4,
                             HI=2, dI=32, k=16, w=16, seed=0, kind="csa"),
    "hca_8k_bf16": Workload("hca_8k_bf16", "bf16", B=2, n=8192, H=16, d=128, r=64,
                            m_hca=128, w=128, seed=1, kind="hca"),
    "csa_prefill_128k": Workload("csa_prefill_128k", "bf16", B=1, n=131072, H=64, d=512,
                                 r=64, m=4, HI=64, dI=128, k=1024, w=128, seed=2,
                                 kind="csa"),
    "decode_256k": Workload("decode_256k", "bf16", B=8, ctx=262144, H=64, d=512, r=64,
                            m=4, m_hca=128, HI=64, dI=128, k=1024, w=128, seed=3,
                            layers=("csa", "hca")),
    "decode_1m": Workload("decode_1m", "bf16", B=4, ctx=1048576, H=64, d=512, r=64, m=4,
                          m_hca=128, HI=64, dI=128, k=1024, w=128, seed=4,
                          layers=("csa", "hca", "csa", "hca"), fp8_keys=True),
    "decode_1m_fp8kv": Workload("decode_1m_fp8kv", "bf16", B=4, ctx=1048576, H=64, d=512, r=64, m=4,
                                m_hca=128, HI=64, dI=128, k=1024, w=128, seed=4,
                                layers=("csa", "hca", "csa", "hca"), fp8_keys=True, fp8_kv=True),
}


class Draw:
    """Deterministic per-tensor draws: tensor ``name`` of a workload always
    comes from the same sub-seed, whatever else is drawn before it."""

    def __init__(self, seed: int, device="cpu"):
        self.seed = int(seed)
        self.device = torch.device(device)

    def _gen(self, name: str) -> torch.Generator:
        h = 1469598103934665603
        for ch in f"{self.seed}/{name}".encode():
            h = ((h ^ ch) * 1099511628211) % (1 << 63)
        g = torch.Generator(device=self.device)
        g.manual_seed(h)
        return g

    def normal(self, name: str, shape, std: float = 1.0, dtype=torch.float32,
               chunk_elems: int = 1 << 28) -> torch.Tensor:
        """N(0, std^2) drawn in fp32, then rounded (RNE) to ``dtype``.
        Large tensors are drawn in chunks to bound the fp32 temporary."""
        g = self._gen(name)
        shape = tuple(int(s) for s in shape)
        numel = math.prod(shape)
        out = torch.empty(numel, dtype=dtype, device=self.device)
        for s in range(0, numel, chunk_elems):
            e = min(numel, s + chunk_elems)
            x = torch.randn(e - s, generator=g, device=self.device, dtype=torch.float32)
            if std != 1.0:
                x.mul_(std)
            out[s:e] = x.to(dtype)
        return out.view(shape)

    def integers(self, name: str, low: int, high: int, shape) -> torch.Tensor:
        g = self._gen(name)
        return torch.randint(low, high, tuple(shape), generator=g, device=self.device)


def quantize_e4m3_rows(x: torch.Tensor, block: int = 128):
    """Per-block e4m3 storage of key rows: scale = amax / 448 per ``block``
    contiguous elements (1 where amax is 0), codes = RNE(x / scale) as
    float8_e4m3fn bytes.  Returns (codes uint8 [..., d], scales f32 [..., d/block])."""
    d = x.shape[-1]
    assert d % block == 0
    xb = x.float().reshape(*x.shape[:-1], d // block, block)
    amax = xb.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (xb / scale[..., None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    codes = q.view(torch.uint8).reshape(x.shape)
    return codes.contiguous(), scale.contiguous()


def kv_fp8_row_bytes(d: int, r: int) -> int:
    """Bytes of an FP8 KV row (the library's layout, include/csahca.h): d - r
    e4m3 codes, r bf16 RoPE dims, (d - r) / 64 fp32 scales, padded to a
    multiple of 128."""
    raw = (d - r) + 2 * r + 4 * ((d - r) // 64)
    return (raw + 127) // 128 * 128


def pack_kv_rows_fp8(x: torch.Tensor, r: int, block: int = 64) -> torch.Tensor:
    """FP8 KV storage of rows x [..., d]: the first d - r dims as e4m3 codes
    with one fp32 scale per `block` of them (quantize_e4m3_rows' rule), the
    last r dims as bf16, then the scales and zero padding.  Returns uint8
    [..., kv_fp8_row_bytes(d, r)]."""
    d = x.shape[-1]
    nr = d - r
    codes, scales = quantize_e4m3_rows(x[..., :nr], block)
    rope = x[..., nr:].to(torch.bfloat16).contiguous().view(torch.uint8)
    sc = scales.to(torch.float32).contiguous().view(torch.uint8)
    row = torch.cat([codes, rope, sc], dim=-1)
    pad = kv_fp8_row_bytes(d, r) - row.shape[-1]
    if pad:
        row = torch.cat([row, torch.zeros(*row.shape[:-1], pad, dtype=torch.uint8, device=row.device)], dim=-1)
    return row.contiguous()


def unpack_kv_rows_fp8(packed: torch.Tensor, d: int, r: int, block: int = 64):
    """The fields of FP8 KV rows: (codes uint8 [..., d-r], scales f32
    [..., (d-r)/block], rope bf16 [..., r])."""
    nr = d - r
    codes = packed[..., :nr]
    rope = packed[..., nr:nr + 2 * r].contiguous().view(torch.bfloat16)
    scales = packed[..., nr + 2 * r:nr + 2 * r + 4 * (nr // block)].contiguous().view(torch.float32)
    return codes, scales, rope


# ----------------------------------------------------------------------------
# per-call input sets
# ----------------------------------------------------------------------------

def compress_inputs(wl: Workload, kind: str, n: int, c: int, seed_tag: str,
                    device="cpu", B: int | None = None):
    """Token streams for one compressor call.

    csa: a, b, za, zb [B, n, c]; bias_a, bias_b [m, c].  hca: a, za [B, n, c];
    bias_a [m', c].  Streams ~ N(0,1)/sqrt(c) (tiny config) or N(0,1) (others);
    logits ~ N(0,1); biases ~ N(0, 0.1^2).
    """
    D = Draw(wl.seed, device)
    B = wl.B if B is None else B
    dt = wl.torch_dtype
    std = 1.0 / math.sqrt(c) if wl.dtype == "f32" else 1.0
    m = wl.m if kind == "csa" else wl.m_hca
    out = {
        "a": D.normal(f"{seed_tag}/Ca", (B, n, c), std, dt),
        "za": D.normal(f"{seed_tag}/Za", (B, n, c), 1.0, dt),
        "bias_a": D.normal(f"{seed_tag}/Ba", (m, c), 0.1, torch.float32),
    }
    if kind == "csa":
        out["b"] = D.normal(f"{seed_tag}/Cb", (B, n, c), std, dt)
        out["zb"] = D.normal(f"{seed_tag}/Zb", (B, n, c), 1.0, dt)
        out["bias_b"] = D.normal(f"{seed_tag}/Bb", (m, c), 0.1, torch.float32)
    return out


def prefill_inputs(wl: Workload, device="cpu", n: int | None = None, B: int | None = None):
    """Everything one prefill layer needs: compressor streams for the KV rows
    (and the indexer keys, CSA), raw per-token window rows, raw queries,
    indexer queries and head weights, sinks and gains (ones)."""
    D = Draw(wl.seed, device)
    n = wl.n if n is None else n
    B = wl.B if B is None else B
    dt = wl.torch_dtype
    tiny = wl.dtype == "f32"
    sd = (1.0 / math.sqrt(wl.d)) if tiny else 1.0
    kind = wl.kind
    inp = {
        "kv": compress_inputs(wl, kind, n, wl.d, "kv", device, B),
        "kv_win": D.normal("kv_win", (B, n, wl.d), sd, dt),
        "q": D.normal("q", (B, n, wl.H, wl.d), sd, dt),
        "sinks": D.normal("sinks", (wl.H,), 1.0, torch.float32),
        "q_gain": torch.ones(wl.d, dtype=torch.float32, device=device),
        "kv_gain": torch.ones(wl.d, dtype=torch.float32, device=device),
    }
    if kind == "csa":
        sdi = (1.0 / math.sqrt(wl.dI)) if tiny else 1.0
        inp["ik"] = compress_inputs(wl, "csa", n, wl.dI, "ik", device, B)
        inp["qI"] = D.normal("qI", (B, n, wl.HI, wl.dI), sdi, dt)
        inp["w"] = D.normal("w", (B, n, wl.HI), 1.0 / math.sqrt(wl.HI), torch.float32)
    return inp


def decode_inputs(wl: Workload, device="cpu", ctx: int | None = None, B: int | None = None,
                  layers=None, room: int = 0):
    """Per-layer decode state and new-token inputs.

    For each layer L: caches already final (Gaussian rows as drawn), with room
    for every entry the new token at position ctx completes, and for those of
    ``room`` further positions: CSA kv [B, (ctx+room+1)/m, d], indexer keys
    [B, (ctx+room+1)/m, d_I] (bf16, or e4m3 codes + fp32 scales), HCA kv
    [B, (ctx+room+1)/m', d]; window ring [B, w, d]; new query
    q [B, H, d] at position ctx, qI [B, H_I, d_I], w [B, H_I]; sinks [H].
    Compressor state and the new token's compressor inputs: ring [B, R, S, d]
    of the raw streams of the R tokens before it (R = 2m, S = 4 for CSA:
    a, b, za, zb; R = m', S = 2 for HCA: a, za), its own streams ca, cb, cza,
    czb (CSA) or ca, cza (HCA) [B, d], its raw window row kv_raw [B, d],
    biases bias_a, bias_b [m, d] ~ N(0, 0.1^2) and kv_gain (ones); for CSA
    the indexer streams ia, ib, iza, izb [B, d_I], iring [B, 2m, 4, d_I] and
    ibias_a, ibias_b [m, d_I].
    """
    D = Draw(wl.seed, device)
    ctx = wl.ctx if ctx is None else ctx
    B = wl.B if B is None else B
    layers = wl.layers if layers is None else layers
    dt = wl.torch_dtype
    out = []
    for li, kind in enumerate(layers):
        t = f"L{li}"
        m = wl.m if kind == "csa" else wl.m_hca
        N = (ctx + room + 1) // m
        L = {
            "kind": kind, "m": m,
            "pos": torch.full((B,), ctx, dtype=torch.int32, device=device),
            "kv": (pack_kv_rows_fp8(D.normal(f"{t}/kv", (B, N, wl.d), 1.0, dt), wl.r) if wl.fp8_kv
                   else D.normal(f"{t}/kv", (B, N, wl.d), 1.0, dt)),
            "win": D.normal(f"{t}/win", (B, wl.w, wl.d), 1.0, dt),
            "q": D.normal(f"{t}/q", (B, wl.H, wl.d), 1.0, dt),
            "sinks": D.normal(f"{t}/sinks", (wl.H,), 1.0, torch.float32),
            "q_gain": torch.ones(wl.d, dtype=torch.float32, device=device),
        }
        if kind == "csa":
            L["qI"] = D.normal(f"{t}/qI", (B, wl.HI, wl.dI), 1.0, dt)
            L["w"] = D.normal(f"{t}/w", (B, wl.HI), 1.0 / math.sqrt(wl.HI), torch.float32)
            kI = D.normal(f"{t}/kI", (B, N, wl.dI), 1.0, dt)
            if wl.fp8_keys:
                codes, scales = quantize_e4m3_rows(kI)
                L["kI"] = codes
                L["kI_scale"] = scales
            else:
                L["kI"] = kI
                L["kI_scale"] = None
        sd = (1.0 / math.sqrt(wl.d)) if wl.dtype == "f32" else 1.0
        S = 4 if kind == "csa" else 2
        R = 2 * m if kind == "csa" else m
        names = ("ca", "cb", "cza", "czb") if kind == "csa" else ("ca", "cza")
        L["ring"] = D.normal(f"{t}/ring", (B, R, S, wl.d), sd, dt)
        for n in names:
            L[n] = D.normal(f"{t}/{n}", (B, wl.d), sd, dt)
        L["kv_raw"] = D.normal(f"{t}/kv_raw", (B, wl.d), sd, dt)
        L["bias_a"] = D.normal(f"{t}/bias_a", (m, wl.d), 0.1, torch.float32)
        L["bias_b"] = D.normal(f"{t}/bias_b", (m, wl.d), 0.1, torch.float32) if kind == "csa" else None
        L["kv_gain"] = torch.ones(wl.d, dtype=torch.float32, device=device)
        if kind == "csa":
            sdi = (1.0 / math.sqrt(wl.dI)) if wl.dtype == "f32" else 1.0
            L["iring"] = D.normal(f"{t}/iring", (B, R, 4, wl.dI), sdi, dt)
            for n in ("ia", "ib", "iza", "izb"):
                L[n] = D.normal(f"{t}/{n}", (B, wl.dI), sdi, dt)
            L["ibias_a"] = D.normal(f"{t}/ibias_a", (m, wl.dI), 0.1, torch.float32)
            L["ibias_b"] = D.normal(f"{t}/ibias_b", (m, wl.dI), 0.1, torch.float32)
        out.append(L)
    return out
