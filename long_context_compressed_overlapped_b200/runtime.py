"""Host runtime around the C ABI: per-rank sharding of decode work, max-over-
ranks timing, a pre-marshalled decode step (all layers of the interleaved
CSA / HCA schedule) and its CUDA-graph capture.

Sharding: decode sequences are independent, so N ranks run N replicas, each on
its own sequences (weak scaling); no collective touches the data path.  The
only collective is the max over ranks of a measured time.
"""

from __future__ import annotations

import ctypes as C
import dataclasses

import torch

from . import api, native, synth


def shard_workload(wl: synth.Workload, rank: int) -> synth.Workload:
    """The workload rank `rank` runs: same shapes, its own sequences (seed)."""
    return dataclasses.replace(wl, seed=wl.seed + 1000 * int(rank))


def max_over_ranks(x: float, group=None) -> float:
    """Max of a per-rank float over the default (or given) process group; x
    itself when torch.distributed is not initialised."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(x)
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend(group) == "nccl" \
        else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


class StepIO:
    """The per-step inputs of every layer (new query, indexer query and
    weights, positions, the new token's compressor streams and raw window
    row) placed in one device arena, and the outputs in
    another: a caller then moves a step's data with one copy each way.  The
    layers' tensors become views of the arenas (same dtype and shape, slots
    256-byte aligned); make the DecodeStep after this."""

    # per layer: the compressors' inputs (and the positions) first, then the attention's
    COMP_NAMES = ("pos", "kv_raw", "ca", "cb", "cza", "czb", "ia", "ib", "iza", "izb")
    IN_NAMES = COMP_NAMES + ("qI", "w", "q")

    def __init__(self, layers, device):
        def arena(tensors):
            offs, off = [], 0
            for t in tensors:
                offs.append(off)
                off = (off + t.numel() * t.element_size() + 255) // 256 * 256
            return torch.empty(max(off, 256), dtype=torch.uint8, device=device), offs

        def view(buf, off, dtype, shape):
            n = 1
            for x in shape:
                n *= x
            nbytes = n * torch.empty((), dtype=dtype).element_size()
            return buf[off:off + nbytes].view(dtype).view(shape)

        ins = [(li, L, n) for li, L in enumerate(layers) for n in self.IN_NAMES if L.get(n) is not None]
        self.inp, offs = arena([L[n] for _, L, n in ins])
        # layer l's inputs and output occupy one contiguous byte range of each
        # arena (the slots are layer-major), so they can move layer by layer;
        # within a layer the compressors' inputs come first (comp_ends[l]:
        # the end of that part)
        self.in_ranges = [[self.inp.numel(), 0] for _ in layers]
        self.comp_ends = [0 for _ in layers]
        for (li, L, n), o in zip(ins, offs):
            v = view(self.inp, o, L[n].dtype, tuple(L[n].shape))
            v.copy_(L[n])
            L[n] = v
            r = self.in_ranges[li]
            end = o + v.numel() * v.element_size()
            r[0], r[1] = min(r[0], o), max(r[1], end)
            if n in self.COMP_NAMES:
                self.comp_ends[li] = max(self.comp_ends[li], end)
        outs = [torch.empty_like(L["q"]) for L in layers]
        self.out, offs = arena(outs)
        self.out_ranges = []
        for L, t, o in zip(layers, outs, offs):
            L["out"] = view(self.out, o, t.dtype, tuple(t.shape))
            self.out_ranges.append((o, o + t.numel() * t.element_size()))


def compress_args(wl: synth.Workload, L, entry_base: int = 0):
    """DecodeCompressArgs of one layer of synth.decode_inputs (and the tensors
    it points to); entry_base: the first global entry of L's cache shard."""
    csa = L["kind"] == "csa"
    streams = tuple(L[n] for n in (("ca", "cb", "cza", "czb") if csa else ("ca", "cza")))
    kw = {}
    if csa:
        kw = dict(istreams=tuple(L[n] for n in ("ia", "ib", "iza", "izb")), ibias_a=L["ibias_a"],
                  ibias_b=L["ibias_b"], iring=L["iring"], kI=L["kI"], kI_scale=L["kI_scale"])
    return api.decode_compress_args(L["kind"], L["pos"], streams, L["ring"], L["kv"], m=L["m"],
                                    bias_a=L["bias_a"], bias_b=L["bias_b"], kv_raw=L["kv_raw"],
                                    win=L["win"], kv_gain=L["kv_gain"], rope_dims=wl.r, entry_base=entry_base,
                                    **kw)


class DecodeStep:
    """One decode step over every layer of `layers` (as made by
    synth.decode_inputs): per layer, the compressors take in the new token
    (decode_compress: ring, window row, a new cache entry when the token
    completes a block), then compressed_attn_decode.  The C-ABI argument
    structs and workspaces are built once, so a call only enqueues the
    library's kernels on `stream`."""

    def __init__(self, wl: synth.Workload, layers, stream: torch.cuda.Stream, keep_idx: bool = False):
        self.lib = native.lib()
        self.stream = stream
        # the layers' tensors were written on the current stream: the step's
        # stream is ordered after that work (later writes are the caller's to order)
        if isinstance(stream, torch.cuda.Stream):
            stream.wait_stream(torch.cuda.current_stream(stream.device))
        self.calls = []
        self.compress = [compress_args(wl, L) for L in layers]
        self.idx = []                            # per layer: the CSA selection (keep_idx) or None
        for L in layers:
            kw = dict(m=L["m"], rope_dims=wl.r, q_gain=L["q_gain"])
            idx = None
            if L["kind"] == "csa":
                if keep_idx:
                    idx = torch.empty(L["q"].shape[0], wl.k, dtype=torch.int32, device=L["q"].device)
                kw.update(k=wl.k, qI=L["qI"], wI=L["w"], kI=L["kI"], kI_scale=L["kI_scale"], idx_out=idx)
            self.idx.append(idx)
            args, out, keep = api.decode_args(L["kind"], L["q"], L["pos"], L["kv"], L["win"],
                                              L["sinks"], out=L.get("out"), **kw)
            nbytes = self.lib.csahca_decode_workspace_size(C.byref(args))
            ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=L["q"].device)
            args.workspace = ws.data_ptr()
            args.workspace_bytes = ws.numel()
            L["out"] = out
            self.calls.append((args, out, keep, ws))
        self.outputs = [c[1] for c in self.calls]

    def compress_step(self, i: int):
        """Enqueue layer i's compressors' step."""
        st = self.lib.decode_compress(C.byref(self.compress[i][0]), self.stream.cuda_stream)
        if st != 0:
            native.check(st, "decode_compress")

    def attention(self, i: int):
        """Enqueue layer i's attention (indexer top-k for CSA, then attention)."""
        st = self.lib.compressed_attn_decode(C.byref(self.calls[i][0]), self.stream.cuda_stream)
        if st != 0:
            native.check(st, "compressed_attn_decode")

    def layer(self, i: int):
        """Enqueue layer i alone: its compressors' step, then its attention."""
        self.compress_step(i)
        self.attention(i)

    def __call__(self):
        for i in range(len(self.calls)):
            self.layer(i)


class DecodeGraph:
    """A DecodeStep captured once into a CUDA graph and replayed: the same
    kernels with the same arguments, without per-launch host work."""

    def __init__(self, step: DecodeStep):
        self.step = step
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(step.stream):
            step()                               # warm the lazy set-up outside capture
        torch.cuda.synchronize()
        with torch.cuda.graph(self.graph, stream=step.stream, capture_error_mode="thread_local"):
            step()
        torch.cuda.synchronize()

    def __call__(self):
        self.graph.replay()


class HostIOGraph:
    """A decode step fed from host memory, captured as one CUDA graph with the
    host copies pipelined: on a copy stream the first layer's compressor
    inputs go first, then its attention inputs, then each later layer's
    slice; the first layer's compressor step waits only for the first part,
    its attention for the second, and each later layer for its own slice
    (which lands while the earlier layers run).  Each layer's output leaves on another
    copy stream as soon as the layer is done.  host_in and host_out are pinned host buffers shaped like
    io.inp and io.out (one host_in per graph: a buffer the host rewrites
    must not be one a replay may still be reading).  Make it after the step
    has run once (the library's first-call set-up happens outside capture)."""

    def __init__(self, step: DecodeStep, io: StepIO, host_in: torch.Tensor, host_out: torch.Tensor):
        self.graph = torch.cuda.CUDAGraph()
        main = step.stream
        cin = torch.cuda.Stream(main.device)
        cout = torch.cuda.Stream(main.device)
        n = len(step.calls)
        a0, b0 = io.in_ranges[0]
        c0 = io.comp_ends[0]
        parts = [(a0, c0), (c0, b0)] + [tuple(r) for r in io.in_ranges[1:]]
        ev_in = [torch.cuda.Event() for _ in parts]
        ev_out = [torch.cuda.Event() for _ in range(n)]

        def enqueue():
            cin.wait_stream(main)
            cout.wait_stream(main)
            with torch.cuda.stream(cin):
                for k, (a, b) in enumerate(parts):
                    if b > a:
                        io.inp[a:b].copy_(host_in[a:b], non_blocking=True)
                    ev_in[k].record(cin)
            for li in range(n):
                if li == 0:
                    main.wait_event(ev_in[0])
                    step.compress_step(0)
                    main.wait_event(ev_in[1])
                    step.attention(0)
                else:
                    main.wait_event(ev_in[li + 1])
                    step.layer(li)
                ev_out[li].record(main)
                cout.wait_event(ev_out[li])
                a, b = io.out_ranges[li]
                with torch.cuda.stream(cout):
                    host_out[a:b].copy_(io.out[a:b], non_blocking=True)
            main.wait_stream(cin)
            main.wait_stream(cout)

        # (capture only: the step has run before, so the library's lazy set-up is done)
        torch.cuda.synchronize()
        with torch.cuda.graph(self.graph, stream=main, capture_error_mode="thread_local"):
            enqueue()
        torch.cuda.synchronize()

    def __call__(self):
        self.graph.replay()
