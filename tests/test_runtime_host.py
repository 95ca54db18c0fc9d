"""Host logic of the decode step, with the library replaced by a recorder (no
GPU, no kernels): per layer the compressor step comes before the attention,
both see the same positions and caches, and the end-to-end arena holds the
new token's compressor inputs."""

import torch

from long_context_compressed_overlapped_b200 import api, native, runtime, synth


class _Recorder:
    def __init__(self):
        self.calls = []

    def decode_compress(self, args, stream):
        a = args._obj
        self.calls.append(("decode_compress", a.kind, a.pos, a.kv_cache, a.win, a.ring, a.kI))
        return 0

    def compressed_attn_decode(self, args, stream):
        a = args._obj
        self.calls.append(("compressed_attn_decode", a.kind, a.pos, a.kv_cache, a.win, None, a.kI))
        return 0

    def csahca_decode_workspace_size(self, args):
        return 256


class _Stream:
    cuda_stream = 0


def test_decode_step_runs_compressor_then_attention_per_layer(monkeypatch):
    rec = _Recorder()
    monkeypatch.setattr(native, "lib", lambda: rec)
    monkeypatch.setattr(api, "_ptr", lambda t: None if t is None else t.data_ptr())
    wl = synth.WORKLOADS["decode_1m"]
    layers = synth.decode_inputs(wl, "cpu", ctx=2047, B=2)
    io = runtime.StepIO(layers, "cpu")
    step = runtime.DecodeStep(wl, layers, _Stream())
    step()
    assert [c[0] for c in rec.calls] == ["decode_compress", "compressed_attn_decode"] * len(wl.layers)
    for li, L in enumerate(layers):
        comp, attn = rec.calls[2 * li], rec.calls[2 * li + 1]
        kind = native.CSA if L["kind"] == "csa" else native.HCA
        assert comp[1] == attn[1] == kind
        assert comp[3] == attn[3] == L["kv"].data_ptr()            # the cache the compressor fills
        assert comp[4] == attn[4] == L["win"].data_ptr()           # the window row it writes
        assert comp[5] == L["ring"].data_ptr()
        if L["kind"] == "csa":
            assert comp[6] == attn[6] == L["kI"].data_ptr()
        # both calls read the positions from the step's input arena
        lo = io.inp.data_ptr()
        assert lo <= comp[2] < lo + io.inp.numel() and comp[2] == attn[2] == L["pos"].data_ptr()
    # the new token's compressor inputs travel in the arena too
    for L in layers:
        for n in ("kv_raw", "ca", "cza"):
            assert io.inp.data_ptr() <= L[n].data_ptr() < io.inp.data_ptr() + io.inp.numel()
    assert torch.equal(layers[0]["pos"], torch.full((2,), 2047, dtype=torch.int32))


def test_step_io_layer_ranges_partition_the_arenas():
    """Layer l's inputs and output lie in one byte range of each arena, the
    ranges in layer order and disjoint: the end-to-end graph moves them layer
    by layer."""
    wl = synth.WORKLOADS["decode_1m"]
    layers = synth.decode_inputs(wl, "cpu", ctx=2047, B=2)
    io = runtime.StepIO(layers, "cpu")
    base_in, base_out = io.inp.data_ptr(), io.out.data_ptr()
    assert len(io.in_ranges) == len(io.out_ranges) == len(layers)
    prev_in = prev_out = 0
    for li, L in enumerate(layers):
        a, b = io.in_ranges[li]
        assert prev_in <= a < b <= io.inp.numel()
        prev_in = b
        c = io.comp_ends[li]
        assert a < c <= b
        for n in runtime.StepIO.IN_NAMES:
            t = L.get(n)
            if t is not None:
                lo = t.data_ptr() - base_in
                hi = lo + t.numel() * t.element_size()
                assert a <= lo and hi <= b, (li, n)
                # the compressors' inputs before comp_ends, the attention's after
                assert (hi <= c) if n in runtime.StepIO.COMP_NAMES else (lo >= c), (li, n)
        a, b = io.out_ranges[li]
        assert prev_out <= a < b <= io.out.numel()
        prev_out = b
        lo = L["out"].data_ptr() - base_out
        assert (a, b) == (lo, lo + L["out"].numel() * L["out"].element_size())
