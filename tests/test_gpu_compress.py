"""GPU parity of csa_compress / hca_compress against the float64 oracle
("Paper Breakdown: DeepSeek-V4", section 4: CSA KV compression, HCA,
Additional Techniques)."""

import numpy as np
import pytest
import torch

from long_context_compressed_overlapped_b200 import api, synth
from tests.helpers import check_close, oracle_compress

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(kind, inp, m, **kw):
    if kind == "csa":
        return api.csa_compress(inp["a"], inp["b"], inp["za"], inp["zb"], inp["bias_a"],
                                inp["bias_b"], m, **kw)
    return api.hca_compress(inp["a"], inp["za"], inp["bias_a"], m, **kw)


@pytest.mark.parametrize("wl_name,kind,n,c,r", [
    ("tiny_csa_f32", "csa", 512 + 3, 64, 16),       # ragged tail of 3 tokens
    ("tiny_csa_f32", "csa", 512, 32, 0),            # indexer keys: no norm, no rope
    ("hca_8k_bf16", "hca", 8192 + 77, 128, 64),
    ("csa_prefill_128k", "csa", 4096 + 2, 512, 64),
    ("csa_prefill_128k", "csa", 4096, 128, 0),      # indexer keys, d_I = 128
])
def test_compress_all_entries(wl_name, kind, n, c, r):
    wl = synth.WORKLOADS[wl_name]
    m = wl.m if kind == "csa" else wl.m_hca
    inp = synth.compress_inputs(wl, kind, n, c, f"t{c}", DEV, B=2)
    rms = r > 0
    gain = torch.linspace(0.5, 1.5, c, device=DEV) if rms else None
    out = _run(kind, inp, m, rms_norm=rms, gain=gain, rope_dims=r)
    assert out.shape == (2, n // m, c)
    ent = np.arange(n // m)
    if len(ent) > 300:
        ent = np.unique(np.concatenate([ent[:40], ent[-40:], np.random.default_rng(0).choice(ent, 100)]))
    for b in range(2):
        ref = oracle_compress(kind, inp, m, b, ent, rms, gain, r)
        check_close(out[b, ent].double().cpu().numpy(), ref, wl.dtype, f"{kind} b={b}")
    assert api.device_error() == 0


def test_compress_block_range():
    """first_block / num_blocks produce exactly the matching slice."""
    wl = synth.WORKLOADS["csa_prefill_128k"]
    inp = synth.compress_inputs(wl, "csa", 1024, 512, "rng", DEV, B=1)
    full = _run("csa", inp, 4, rope_dims=64)
    part = _run("csa", inp, 4, rope_dims=64, first_block=37, num_blocks=11)
    assert torch.equal(part, full[:, 37:48])
    one = _run("csa", inp, 4, rope_dims=64, first_block=0, num_blocks=1)
    assert torch.equal(one, full[:, :1])


@pytest.mark.slow
def test_compress_full_size_sampled():
    """csa_prefill_128k at full size (n = 131072, d = 512) on sampled entries."""
    wl = synth.WORKLOADS["csa_prefill_128k"]
    inp = synth.compress_inputs(wl, "csa", wl.n, wl.d, "kv", DEV, B=1)
    out = _run("csa", inp, wl.m, rope_dims=wl.r)
    ent = np.unique(np.r_[0, 1, 2, wl.n // wl.m - 1, np.random.default_rng(1).choice(wl.n // wl.m, 60)])
    ref = oracle_compress("csa", inp, wl.m, 0, ent, True, None, wl.r)
    check_close(out[0, ent].double().cpu().numpy(), ref, "bf16", "full-size csa")
    assert api.device_error() == 0
