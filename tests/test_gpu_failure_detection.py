"""The failure path of the bounded device waits, on the GPU, without a
fault: a kernel waits on a barrier that nothing completes, its bounded wait
gives up, the device error word reports it (code 1) and is cleared, and the
context stays usable (the next call runs and matches the oracle)."""

import time

import numpy as np
import pytest

from long_context_compressed_overlapped_b200 import api, synth
from tests.helpers import check_close, oracle_compress

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_bounded_wait_gives_up_and_the_device_stays_usable():
    assert api.device_error() == 0
    t0 = time.monotonic()
    api.selftest_bounded_wait()
    code = api.device_error()
    waited = time.monotonic() - t0
    assert code == 1, f"device error word {code}"
    assert waited < 5.0, f"the bounded wait took {waited:.1f} s"
    assert api.device_error() == 0, "reading the word clears it"
    # a call after the give-up runs normally
    wl = synth.WORKLOADS["tiny_csa_f32"]
    inp = synth.compress_inputs(wl, "csa", 256 + 3, 64, "t64", DEV, B=1)
    out = api.csa_compress(inp["a"], inp["b"], inp["za"], inp["zb"], inp["bias_a"], inp["bias_b"], wl.m,
                           rms_norm=True, rope_dims=16)
    ent = np.arange(out.shape[1])
    ref = oracle_compress("csa", inp, wl.m, 0, ent, True, None, 16)
    check_close(out[0].double().cpu().numpy(), ref, wl.dtype, "csa after a given-up wait")
    assert api.device_error() == 0
