"""The N > 1 path on CPU: two gloo ranks.  Each rank runs its own sequences
(weak scaling, different seeds, same shapes) and the timing reduction is the
max over ranks; no collective touches the data."""

import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_compressed_overlapped_b200 import runtime, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = runtime.shard_workload(synth.WORKLOADS["decode_1m"], rank)
        layers = synth.decode_inputs(wl, "cpu", ctx=2048, B=2, layers=("csa", "hca"))
        fingerprint = float(layers[0]["q"].float().sum())
        t = runtime.max_over_ranks(10.0 + rank)
        gathered = [None] * world
        dist.all_gather_object(gathered, (wl.seed, fingerprint, tuple(layers[0]["kv"].shape)))
        q.put((rank, t, gathered))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, gathered in res:
        assert t == 11.0                                  # max over ranks
        seeds = [g[0] for g in gathered]
        assert len(set(seeds)) == world                   # each rank: its own sequences
        assert len({g[1] for g in gathered}) == world     # different data
        assert len({g[2] for g in gathered}) == 1         # same shapes (weak scaling)


def test_single_process_max_is_identity():
    assert runtime.max_over_ranks(3.5) == 3.5


def test_step_io_arenas_hold_every_input_and_output():
    """StepIO moves each layer's per-step inputs into one arena (same values,
    dtypes and shapes, 256-byte aligned slots) and gives every layer an output
    view of a second arena: a step's data then moves with one copy each way."""
    g = torch.Generator().manual_seed(0)
    layers = [
        dict(q=torch.randn(4, 64, 512, generator=g).bfloat16(), qI=torch.randn(4, 64, 128, generator=g).bfloat16(),
             w=torch.randn(4, 64, generator=g), pos=torch.arange(4, dtype=torch.int32)),
        dict(q=torch.randn(4, 64, 512, generator=g).bfloat16(), pos=torch.arange(4, 8, dtype=torch.int32)),
    ]
    ref = [{k: v.clone() for k, v in L.items()} for L in layers]
    io = runtime.StepIO(layers, "cpu")
    base_in, base_out = io.inp.data_ptr(), io.out.data_ptr()
    for L, R in zip(layers, ref):
        for k, v in R.items():
            assert torch.equal(L[k], v) and L[k].dtype == v.dtype and L[k].shape == v.shape
            off = L[k].data_ptr() - base_in
            assert 0 <= off < io.inp.numel() and off % 256 == 0
        off = L["out"].data_ptr() - base_out
        assert L["out"].shape == R["q"].shape and 0 <= off < io.out.numel() and off % 256 == 0
    # the arena is the data: writing it changes the layers' inputs
    io.inp.zero_()
    assert all(float(L["q"].float().abs().sum()) == 0.0 for L in layers)
