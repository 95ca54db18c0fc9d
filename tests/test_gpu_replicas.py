"""The bench's N > 1 path with the library on the GPU: two ranks (gloo for
the exchange, both on this machine's one GPU, taking turns) each run a decode
step of their own sequences (runtime.shard_workload: same shapes, the rank's
own seed) and check it against the oracle; the timing reduction is the max
over ranks.  The ranks' kernels never wait on one another: replicas share no
data."""

import os
import socket
import traceback

import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from long_context_compressed_overlapped_b200 import api, runtime, synth
        from tests.test_gpu_decode import _check_layer, _decode_layer
        torch.cuda.set_device(0)
        wl = runtime.shard_workload(synth.WORKLOADS["decode_256k"], rank)
        ctx = 8192 + 5
        layers = synth.decode_inputs(wl, "cuda", ctx=ctx, B=2)
        fingerprint = float(layers[0]["q"].float().sum())
        torch.cuda.synchronize()
        err = None
        # the ranks take turns on the GPU: two contexts never time-slice the
        # scan's waits for its own co-resident CTAs
        for turn in range(world):
            if turn == rank:
                for L in layers:
                    idx = torch.empty(2, wl.k, dtype=torch.int32, device="cuda") if L["kind"] == "csa" else None
                    out = _decode_layer(L, wl, idx_out=idx)
                    _check_layer(L, wl, out, idx, range(2))
                err = api.device_error()
            dist.barrier()
        t = runtime.max_over_ranks(10.0 + rank)
        gathered = [None] * world
        dist.all_gather_object(gathered, (wl.seed, fingerprint, err))
        q.put((rank, t, gathered, None))
    except Exception:                                       # reported to the parent
        q.put((rank, None, None, traceback.format_exc()))
    finally:
        dist.destroy_process_group()


def test_two_replica_ranks_match_the_oracle():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=600) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    for rank, t, gathered, exc in res:
        assert exc is None, f"rank {rank}:\n{exc}"
        assert t == 11.0                                   # max over ranks
        assert len({g[0] for g in gathered}) == world      # each rank: its own sequences
        assert len({g[1] for g in gathered}) == world      # different data
        assert all(g[2] == 0 for g in gathered)            # no device error on either rank
    assert all(p.exitcode == 0 for p in procs)
