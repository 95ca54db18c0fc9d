#!/usr/bin/env python
"""Throughput of the CSA + HCA compressed-attention hot path on B200.

One step = one decode step of the decode_1m workload through the C ABI:
4 sequences x 4 layers (CSA, HCA, CSA, HCA) at a cached context of about
1,048,576 tokens (CSA 4:1 with e4m3 indexer keys and top-1024, HCA 128:1
dense, 128-token window, 64 heads of 512 dims).  The K timed steps take
consecutive positions, so the compressors complete a CSA block every fourth
step and one HCA block mid-run, as in a real decode.  `value` = tokens/s over
all ranks (each rank runs its own 4 sequences: weak scaling, no collective on
the data path).  The line also carries the decode_256k workload (8 sequences,
one CSA + one HCA layer at 262,144 tokens) and the csa_prefill_128k layer (one
CSA prefill of 131,072 tokens: both compressors, indexer top-k, attention)
against the sustained dense bf16 peak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--no-prefill] [--no-256k]

--impl reference times the float64 CPU oracle (the only reference that
exists for this path) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import ctypes as C
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_compressed_overlapped_b200 import api, native, runtime, synth  # noqa: E402

METRIC = "CSA+HCA attention tokens/s (decode@1M, prefill@128K); % HBM / TC roofline"
L2_BYTES = 126 * 2**20


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ------------------------------------------------------------ distributed ----

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    return runtime.max_over_ranks(x) if world > 1 else x


# ------------------------------------------------------------------ clocks ----

class ClockSampler:
    """SM clock and throttle reasons of this GPU, sampled through NVML every
    2 ms by a host thread while the timed loop runs (nvidia-smi reads the same
    counters; its 200 ms period is too coarse for a timed region of tens of
    milliseconds).  Falls back to nvidia-smi -lms 200 if NVML is unavailable."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device: int, period_s: float = 0.002):
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.handle = None
        self.thread = None
        self.proc = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
        except Exception:
            self.handle = None

    def _loop(self):
        n = self.nvml
        while not self.stop_flag.is_set():
            try:
                self.samples.append(float(n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)))
                bits = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                for name, bit in self.REASONS.items():
                    if bits & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        self.samples, self.reasons = [], set()
        if self.handle is not None:
            self.stop_flag = threading.Event()
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
            return
        try:
            self.path = tempfile.mktemp(prefix="clocks_", suffix=".csv")
            self.fh = open(self.path, "w")
            cmd = ["nvidia-smi", "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                   "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                   "clocks_event_reasons.sw_power_cap", "--format=csv,noheader,nounits", "-lms", "200"]
            self.proc = subprocess.Popen(cmd, stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join()
            src = "nvml"
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            with open(self.path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    try:
                        self.samples.append(float(parts[0]))
                        self.max_mhz = float(parts[1])
                    except (ValueError, IndexError):
                        continue
                    for nm, val in zip(names, parts[2:6]):
                        if val.lower().startswith("active"):
                            self.reasons.add(nm)
            os.unlink(self.path)
            src = "nvidia-smi"
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"], "samples": 0}
        sm = self.samples
        busy = [x for x in sm if self.max_mhz and x > 0.5 * self.max_mhz] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(sm), "source": src}


# ------------------------------------------------------- committed ncu data ----

def ncu_traffic(kernel_name):
    """DRAM bytes per launch of `kernel_name` from the committed ncu summary
    (profiles/*.md lines `kernel:`, `source_sha256:`, `dram_bytes_per_launch:`),
    used only while the kernel's source file still has the hash the capture
    was taken with; None otherwise."""
    import glob
    import hashlib
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        meta = {}
        with open(path) as f:
            for line in f:
                if ":" in line and line.split(":", 1)[0].strip() in ("kernel", "source", "source_sha256",
                                                                      "dram_bytes_per_launch"):
                    k_, v_ = line.split(":", 1)
                    meta[k_.strip()] = v_.strip().strip("`")
        if meta.get("kernel") != kernel_name or "source" not in meta:
            continue
        src = os.path.join(ROOT, meta["source"])
        if not os.path.exists(src):
            continue
        with open(src, "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != meta.get("source_sha256"):
                continue
        try:
            return float(meta["dram_bytes_per_launch"])
        except (KeyError, ValueError):
            return None
    return None


# ----------------------------------------------------------- decode step ----

def decode_bytes_per_kernel(wl, ctx):
    """Algorithmic bytes per launch of each traced decode kernel (one launch
    covers the B sequences of one layer)."""
    B, d, H, HI, dI, k, w = wl.B, wl.d, wl.H, wl.HI, wl.dI, wl.k, wl.w
    vc = (ctx + 1) // wl.m
    vh = (ctx + 1) // wl.m_hca
    key_row = dI + 4 * (dI // 128) if wl.fp8_keys else 2 * dI
    # a cache row: d bf16, or (FP8 KV) d - r codes + r bf16 + (d - r) / 64 fp32 scales
    kv_row = (d - wl.r) + 2 * wl.r + 4 * ((d - wl.r) // 64) if wl.fp8_kv else 2 * d
    qo = 2 * H * d * 2
    return {
        "indexer_scores": B * (vc * key_row + HI * dI * 2 + HI * 4),
        "topk_rows": B * (vc * 4 + k * 4),
        "attn_decode_csa": B * (k * kv_row + w * d * 2 + qo),
        "attn_decode_hca": B * (vh * kv_row + w * d * 2 + qo),
        "decode_compress": sum(decode_compress_bytes(wl, kd, ctx) for kd in wl.layers) / len(wl.layers),
    }


def decode_compress_bytes(wl, kind, pos):
    """Algorithmic bytes of one decode_compress launch (B sequences, new token
    at `pos`): the token's raw streams read and stored in the ring, its raw
    window row read and the finished row written; when the token completes a
    block, the other tokens of the pooled blocks (value and logit streams)
    are read and the entry (and its indexer key) written."""
    es = 4 if wl.dtype == "f32" else 2
    m = wl.m if kind == "csa" else wl.m_hca
    S = 4 if kind == "csa" else 2
    per = 2 * S * wl.d * es + 2 * wl.d * es
    if kind == "csa":
        per += 2 * 4 * wl.dI * es
    if (pos + 1) % m == 0:
        i = (pos + 1) // m - 1
        J = m if (kind == "hca" or i == 0) else 2 * m
        kv_row = (wl.d - wl.r) + 2 * wl.r + 4 * ((wl.d - wl.r) // 64) if wl.fp8_kv else wl.d * es
        per += (J - 1) * 2 * wl.d * es + kv_row
        if kind == "csa":
            key = wl.dI + 4 * (wl.dI // 128) if wl.fp8_keys else wl.dI * es
            per += (J - 1) * 2 * wl.dI * es + key
    return wl.B * per


def decode_step_bytes(wl, ctx):
    """Algorithmic HBM bytes of one whole decode step (all layers)."""
    per = decode_bytes_per_kernel(wl, ctx)
    tot = 0
    for kind in wl.layers:
        tot += decode_compress_bytes(wl, kind, ctx)
        if kind == "csa":
            tot += per["indexer_scores"] + per["attn_decode_csa"]
        else:
            tot += per["attn_decode_hca"]
    return tot


def kernel_bytes_key(name):
    if name.startswith("indexer_scores"):
        return "indexer_scores"
    if name.startswith("topk"):
        return "topk_rows"
    if "decode_csa" in name:
        return "attn_decode_csa"
    if "decode_hca" in name:
        return "attn_decode_hca"
    if name.startswith("decode_compress"):
        return "decode_compress"
    return None


def time_steps(step, K, stream, between, world):
    """K steps, each bracketed by CUDA events on `stream`; between(i) runs
    before step i outside the events (L2 flush, position of the step).
    Returns (max over ranks of the summed device time in ms, per-step ms of
    this rank)."""
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(K):
            between(i)
            starts[i].record(stream)
            step()
            ends[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return max_over_ranks(sum(per), world), per


def run_start(wl, K):
    """First position of a run of K consecutive decode steps: the cached
    context is wl.ctx tokens or a few more, CSA blocks complete at every
    fourth step and one HCA block (position = -1 mod m') completes in the
    middle of the run."""
    mh = wl.m_hca
    return wl.ctx + mh - (K + 1) // 2 - (wl.ctx % mh) if K < mh else wl.ctx


def step_kind(wl, pos):
    """Which compressors complete a block at this position."""
    hca = any(k == "hca" for k in wl.layers) and (pos + 1) % wl.m_hca == 0
    csa = any(k == "csa" for k in wl.layers) and (pos + 1) % wl.m == 0
    return "csa_and_hca_block" if (csa and hca) else "hca_block" if hca else "csa_block" if csa else "no_block"


def decode_run(wl, args, dev, stream, world, rank, want_cpu, e2e=True):
    """Time K consecutive decode steps of workload `wl` (all its layers and
    sequences) through the C ABI, launched as one CUDA graph per step; a
    second, traced pass gives the per-kernel times; optionally the same run
    end to end from host buffers, and the oracle on the host."""
    K = args.steps
    p0 = run_start(wl, K)
    positions = [p0 + i for i in range(K)]
    layers = synth.decode_inputs(runtime.shard_workload(wl, rank), dev, ctx=p0, room=K)
    io = runtime.StepIO(layers, dev)            # per-step inputs / outputs in one arena each
    layers_host = host_layers(layers) if want_cpu else None   # the oracle's copy, before any kernel
    # the inputs are made on the current stream; the step runs on `stream`
    torch.cuda.synchronize()
    eager = runtime.DecodeStep(wl, layers, stream)
    step = eager if args.no_graph else runtime.DecodeGraph(eager)
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def set_pos(p):
        for L in layers:
            L["pos"].fill_(p)

    def between(i):
        flush_buf.random_(0, 255)
        set_pos(positions[i % K])

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            between(i)
            step()
    torch.cuda.synchronize()
    if api.device_error(stream) != 0:
        raise RuntimeError("device error flag set during warm-up")

    clocks = ClockSampler(dev.index)
    clocks.start()
    total_ms, per_step = time_steps(step, K, stream, between, world)
    clk = clocks.stop()
    ms_per_step = total_ms / K
    tokens = world * wl.B * K
    value = tokens / (total_ms / 1000.0)
    kinds = {}
    for p, ms in zip(positions, per_step):
        kinds.setdefault(step_kind(wl, p), []).append(ms)

    # traced pass: per-kernel device time of the same K steps (eager launches,
    # so every kernel is bracketed by its own events)
    api.trace_enable(True)
    time_steps(eager, K, stream, between, world)
    traced = api.trace_collect()
    api.trace_enable(False)

    pk = peaks()
    per_pos = [decode_bytes_per_kernel(wl, p) for p in positions]
    per_bytes = {k_: sum(d[k_] for d in per_pos) / K for k_ in per_pos[0]}
    dom = max(traced.items(), key=lambda kv: kv[1][1])
    dname, (dl, dms) = dom
    key = kernel_bytes_key(dname)
    roof = None
    if key is not None:
        ach = per_bytes[key] / (dms / dl / 1000.0) / 1e9
        roof = {"kernel": dname, "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": ach / pk["hbm_gbs"], "traffic": ncu_traffic(dname),
                "peak_source": pk["source"], "launches": dl, "avg_us": 1000 * dms / dl}
    step_bytes = sum(decode_step_bytes(wl, p) for p in positions) / K
    step_frac = step_bytes / (ms_per_step / 1000.0) / 1e9 / pk["hbm_gbs"]
    out = {
        "value": value, "ms_per_step": ms_per_step, "tokens_per_step": world * wl.B,
        "positions": [positions[0], positions[-1]],
        "ms_per_step_by_kind": {k_: {"steps": len(v), "ms": sum(v) / len(v)} for k_, v in sorted(kinds.items())},
        "roofline": roof,
        "step_hbm": {"algorithmic_bytes": step_bytes, "frac": step_frac, "peak": pk["hbm_gbs"],
                     "peak_source": pk["source"]},
        "clocks": clk,
        "gpu_launches": sum(v[0] for v in traced.values()) // K * K,
        "kernels_ms_per_step": {k_: v[1] / K for k_, v in traced.items()},
        "launch": "eager" if args.no_graph else "cuda_graph",
    }

    if e2e:
        # end to end: each step's inputs (positions included) copied in from
        # pinned host memory and its outputs read back, one copy each way
        # (the layers' tensors are views of the two arenas)
        host_inps = []
        for p in positions:
            set_pos(p)
            host_inps.append(io.inp.cpu().pin_memory())
        host_outp = torch.empty(io.out.shape, dtype=io.out.dtype).pin_memory()
        h2d, d2h = io.inp.numel(), io.out.numel()
        state = {"i": 0}
        # one graph per step's host buffer: the copies pipelined layer by layer
        # with the kernels (runtime.HostIOGraph)
        graphs = [runtime.HostIOGraph(eager, io, h, host_outp) for h in host_inps]

        def e2e_between(i):
            flush_buf.random_(0, 255)
            state["i"] = i

        def e2e_step():
            graphs[state["i"] % K]()

        with torch.cuda.stream(stream):
            e2e_step()
        torch.cuda.synchronize()
        e2e_ms, _ = time_steps(e2e_step, K, stream, e2e_between, world)
        out["e2e"] = {"value": tokens / (e2e_ms / 1000.0), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h}
    if api.device_error(stream) != 0:
        raise RuntimeError("device error flag set during the timed region")
    if want_cpu:
        out["cpu_baseline"] = cpu_baseline(wl, layers_host)
    del step, eager
    return out


# -------------------------------------------------------------- prefill ----

def prefill_layer_fn(wl, dev, stream):
    """One csa_prefill_128k layer through the C ABI: both compressors, the
    indexer top-k and the attention.  Returns (step, inputs, state) where
    state holds the last step's compressed rows, indexer keys and output."""
    inp = synth.prefill_inputs(wl, dev)
    kvi, ik = inp["kv"], inp["ik"]
    q_pos = torch.arange(wl.n, device=dev, dtype=torch.int32)[None].repeat(wl.B, 1).contiguous()
    idx = torch.empty(wl.B, wl.n, wl.k, dtype=torch.int32, device=dev)
    out = torch.empty_like(inp["q"])
    state = {"idx": idx, "out": out}

    def step():
        with torch.cuda.stream(stream):
            kv = api.csa_compress(kvi["a"], kvi["b"], kvi["za"], kvi["zb"], kvi["bias_a"],
                                  kvi["bias_b"], wl.m, gain=inp["kv_gain"], rope_dims=wl.r,
                                  stream=stream)
            kI = api.csa_compress(ik["a"], ik["b"], ik["za"], ik["zb"], ik["bias_a"],
                                  ik["bias_b"], wl.m, rms_norm=False, stream=stream)
            api.indexer_topk(inp["qI"], inp["w"], kI, q_pos, wl.m, wl.k, idx=idx, stream=stream)
            api.compressed_attn_prefill("csa", inp["q"], kv, inp["kv_win"], inp["sinks"], m=wl.m,
                                        w=wl.w, rope_dims=wl.r, idx=idx, q_gain=inp["q_gain"],
                                        kv_gain=inp["kv_gain"], out=out, stream=stream)
            state["kv"], state["kI"] = kv, kI
    return step, inp, state


def prefill_flops(wl):
    n, m, k, w = wl.n, wl.m, wl.k, wl.w
    t = np.arange(n, dtype=np.int64)
    vis = (t + 1) // m
    pairs = int(vis.sum())
    keys = int(np.minimum(vis, k).sum() + np.minimum(w, t + 1).sum())
    idx_fl = pairs * wl.HI * wl.dI * 2
    att_fl = keys * wl.H * wl.d * 4
    return idx_fl, att_fl


def prefill_row_flops(wl, t):
    """Algorithmic flops of query t (indexer over its visible entries plus
    attention over its selected entries and window)."""
    v = (t + 1) // wl.m
    return v * wl.HI * wl.dI * 2 + (min(v, wl.k) + min(wl.w, t + 1)) * wl.H * wl.d * 4


def prefill_kernel_flops(name, idx_fl, att_fl):
    if name.startswith("indexer_scores_tc_prefill"):
        return idx_fl
    if name.startswith("attn_prefill"):
        return att_fl
    return None


def prefill_run(args, dev, stream, world, want_cpu):
    """Time the csa_prefill_128k layer (compressors, indexer top-k, attention)
    with per-kernel events; roofline against the sustained dense bf16 peak."""
    pw = synth.WORKLOADS["csa_prefill_128k"]
    pstep, inp, state = prefill_layer_fn(pw, dev, stream)
    torch.cuda.synchronize()                    # inputs made on the current stream; the layer runs on `stream`
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    # warm-up layers with the launch trace on, so that its event pool exists
    # before the timed layers (a first traced layer measured 15-70 ms slower)
    api.trace_enable(True)
    for _ in range(max(3, args.warmup)):
        flush_buf.random_(0, 255)
        with torch.cuda.stream(stream):
            pstep()
    torch.cuda.synchronize()
    api.trace_collect()
    p_ms, _ = time_steps(pstep, args.prefill_steps, stream, lambda i: flush_buf.random_(0, 255), world)
    ptr = api.trace_collect()
    api.trace_enable(False)
    if api.device_error(stream) != 0:
        raise RuntimeError("device error flag set during the prefill run")
    idx_fl, att_fl = prefill_flops(pw)
    tot_fl = idx_fl + att_fl
    pk = peaks()
    peak_tf = pk["bf16_tflops_sustained"]
    ms_layer = p_ms / args.prefill_steps
    kernels = {k_: {"launches_per_layer": v[0] / args.prefill_steps, "ms_per_layer": v[1] / args.prefill_steps}
               for k_, v in ptr.items()}
    dname, (dl, dms) = max(ptr.items(), key=lambda kv: kv[1][1])
    dfl = prefill_kernel_flops(dname, idx_fl, att_fl)
    roof = None
    if dfl is not None:
        ach = dfl / (dms / args.prefill_steps / 1000.0) / 1e12
        roof = {"kernel": dname, "bound": "tensor", "achieved": ach, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": ach / peak_tf, "traffic": ncu_traffic(dname), "peak_source": pk["source"] + " (sustained)",
                "flops_per_layer": dfl, "ms_per_layer": dms / args.prefill_steps}
    out = {"workload": pw.name, "value": world * pw.n / (ms_layer / 1000), "unit": "tokens/s",
           "ms_per_layer": ms_layer, "steps": args.prefill_steps,
           "tflops": tot_fl / (ms_layer / 1000) / 1e12,
           "frac_of_bf16_peak": tot_fl / (ms_layer / 1000) / 1e12 / peak_tf,
           "peak_tflops": peak_tf, "peak_source": pk["source"] + " (sustained)",
           "algorithmic_flops": tot_fl, "roofline": roof,
           "gpu_launches": sum(v[0] for v in ptr.values()),
           "kernels": kernels}
    if want_cpu:
        out["cpu_baseline"] = prefill_cpu_baseline(pw, inp, state)
    return out


# ------------------------------------------------------------ CPU oracle ----

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def oracle_decode_sequence(wl, layers, b, sels=None, scores_out=None):
    """The oracle's decode step for sequence b over all layers: per layer the
    compressor step (new token into the ring, its window row, a new entry
    when it completes a block), then the indexer top-k (CSA) and attention.
    sels: optional per-layer selections used instead of the oracle's own
    top-k (None entries keep it); scores_out: a list that receives each CSA
    layer's indexer scores."""
    from oracle import csahca_oracle as O

    def npy(t):
        return t.detach().cpu().to(torch.float64).numpy() if t.dtype != torch.uint8 else t.cpu().numpy()

    outs = []
    for li, L in enumerate(layers):
        pos = int(L["pos"][b])
        csa = L["kind"] == "csa"
        m = L["m"]
        names = ("a", "b", "za", "zb") if csa else ("a", "za")
        cols = ("ca", "cb", "cza", "czb") if csa else ("ca", "cza")
        ring = {s_: npy(L["ring"][b, :, j]) for j, s_ in enumerate(names)}
        new = {s_: npy(L[c_][b]) for s_, c_ in zip(names, cols)}
        biases = (npy(L["bias_a"]), npy(L["bias_b"]) if csa else None)
        _, entry, win_row = O.decode_compress_step(L["kind"], pos, new, ring, biases, m,
                                                   kv_raw=npy(L["kv_raw"][b]), gain=npy(L["kv_gain"]),
                                                   r=wl.r)
        win = npy(L["win"][b])
        win[pos % wl.w] = win_row
        fp8_kv = L["kv"].dtype == torch.uint8
        if fp8_kv:
            # the rows an FP8 KV cache stands for, and the new entry as stored
            kv = O.dequant_kv_rows_fp8(*(npy(t_) for t_ in synth.unpack_kv_rows_fp8(L["kv"][b], wl.d, wl.r)))
        else:
            kv = npy(L["kv"][b])
        N_cap = kv.shape[0]
        if entry is not None and entry[0] < N_cap:
            kv[entry[0]] = O.dequant_kv_rows_fp8(*O.quantize_kv_rows_fp8(entry[2], wl.r)) if fp8_kv else entry[2]
        sel = None
        if csa:
            v = min(O.n_visible(pos, m), N_cap)
            if L["kI_scale"] is not None:
                K = O.dequant_e4m3_rows(npy(L["kI"][b, :v]), npy(L["kI_scale"][b, :v]))
            else:
                K = npy(L["kI"][b, :v])
            iring = {s_: npy(L["iring"][b, :, j]) for j, s_ in enumerate(names)}
            inew = {s_: npy(L[c_][b]) for s_, c_ in zip(names, ("ia", "ib", "iza", "izb"))}
            _, ientry, _ = O.decode_compress_step("csa", pos, inew, iring,
                                                  (npy(L["ibias_a"]), npy(L["ibias_b"])), m,
                                                  normalize=False)
            if ientry is not None and ientry[0] < v:
                key = ientry[1]
                if L["kI_scale"] is not None:
                    codes, scales = O.quantize_e4m3_rows_f32(key)
                    key = O.dequant_e4m3_rows(codes, scales)
                K[ientry[0]] = key
            s = O.indexer_scores(npy(L["qI"][b]), npy(L["w"][b]), K)
            if scores_out is not None:
                scores_out.append(s)
            sel = O.top_k_select(s, wl.k)
            if sels is not None and sels[li] is not None:
                sel = np.asarray(sels[li])
        outs.append(O.decode_attention(L["kind"], npy(L["q"][b]), pos, kv, win, npy(L["sinks"]),
                                       m=m, w=wl.w, r=wl.r, q_gain=npy(L["q_gain"]), sel=sel))
    return outs


def host_layers(layers):
    """Host copies of the layer tensors the oracle reads (one sequence's worth
    is sliced later)."""
    out = []
    for L in layers:
        H = {}
        for k_, v in L.items():
            H[k_] = v.cpu() if isinstance(v, torch.Tensor) else v
        out.append(H)
    return out


def cpu_baseline(wl, layers_host, budget_s=12.0):
    """Oracle decode steps on whole sequences until ~budget_s of CPU work."""
    t0 = time.perf_counter()
    seqs = 0
    while True:
        oracle_decode_sequence(wl, layers_host, seqs % wl.B)
        seqs += 1
        if time.perf_counter() - t0 >= budget_s or seqs >= wl.B:
            break
    el = time.perf_counter() - t0
    return {"value": seqs / el, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{seqs} of {wl.B} sequences of one decode step, all {len(wl.layers)} layers "
                      f"(float64 NumPy, {el:.1f} s)"}


def prefill_cpu_baseline(pw, inp, state, rows=2048, entries=4096):
    """The oracle on a bounded sample of the csa_prefill_128k layer,
    extrapolated to the whole layer: both compressors on their first
    `entries` entries, then for `rows` seeded queries (uniform over t) the
    indexer scores over every visible entry, the top-k and the attention over
    the selection and the window.  The compressor time scales by
    N_c / entries, the query time by the ratio of the algorithmic flops of
    all n queries to those of the sample."""
    from oracle import csahca_oracle as O

    def npy(t):
        return t.detach().cpu().to(torch.float64).numpy()

    m, n = pw.m, pw.n
    toks = slice(0, entries * m)
    comp_in = [tuple(npy(st[k_][0, toks]) for k_ in ("a", "b", "za", "zb")) + (npy(st["bias_a"]), npy(st["bias_b"]))
               for st in (inp["kv"], inp["ik"])]
    ts = np.sort(np.random.default_rng(2).choice(n, rows, replace=False))
    sel_t = torch.as_tensor(ts, device=inp["q"].device)
    KI, KV = npy(state["kI"][0]), npy(state["kv"][0])
    qI, w = npy(inp["qI"][0].index_select(0, sel_t)), npy(inp["w"][0].index_select(0, sel_t))
    q = npy(inp["q"][0].index_select(0, sel_t))
    kv_win = npy(inp["kv_win"][0])
    sinks, qg, kg = npy(inp["sinks"]), npy(inp["q_gain"]), npy(inp["kv_gain"])
    t0 = time.perf_counter()
    for j, args_ in enumerate(comp_in):
        pooled = O.csa_pool(*args_, m)
        if j == 0:
            O.finish_rows(pooled, np.arange(pooled.shape[0]) * m, kg, pw.r)
    t_comp = time.perf_counter() - t0
    t1 = time.perf_counter()
    for j, t in enumerate(ts):
        t = int(t)
        sc = O.indexer_scores(qI[j], w[j], KI[: O.n_visible(t, m)])
        sel = O.top_k_select(sc, pw.k)
        O.prefill_attention("csa", q[j:j + 1], KV, kv_win, sinks, m=m, w=pw.w, r=pw.r, q_gain=qg,
                            kv_gain=kg, idx={t: sel}, rows=[t], q_holds_rows=True)
    t_rows = time.perf_counter() - t1
    idx_fl, att_fl = prefill_flops(pw)
    sample_fl = sum(prefill_row_flops(pw, int(t)) for t in ts)
    n_c = n // m
    est = t_comp * n_c / entries + t_rows * (idx_fl + att_fl) / sample_fl
    return {"value": pw.B * n / est, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "extrapolated": True, "measured_s": t_comp + t_rows,
            "sample": f"extrapolated: both compressors on {entries} of {n_c} entries (x{n_c // entries}) and "
                      f"{rows} seeded queries of {n} (indexer, top-k, attention; scaled by the algorithmic "
                      f"flop ratio {(idx_fl + att_fl) / sample_fl:.0f}), float64 NumPy, "
                      f"{t_comp + t_rows:.1f} s measured"}


# ------------------------------------------------------------------ main ----

def run_reference(args, world, rank):
    """Reference arm: the float64 oracle on the host cores (rank 0 only).
    A step is one bounded sample of the decode step: one layer of one
    sequence (a quarter of a token with four layers), cycling over every
    layer of every sequence, so that the default run ends within minutes."""
    if rank != 0:
        return
    wl = synth.WORKLOADS[args.workload]
    layers = synth.decode_inputs(wl, "cpu" if not torch.cuda.is_available() else "cuda")
    layers_host = host_layers(layers)
    del layers
    nl = len(wl.layers)

    def sample(i):
        oracle_decode_sequence(wl, [layers_host[i % nl]], (i // nl) % wl.B)

    for i in range(args.warmup):
        sample(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        sample(i)
    el = time.perf_counter() - t0
    value = args.steps / nl / el                    # each sample is 1/nl of a token's layers
    cores = blas_threads()
    what = f"one layer of one sequence per step, cycling over the {nl} layers of the {wl.B} sequences"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "global_batch": 1, "seq_len": wl.ctx, "layers": list(wl.layers),
                   "sample": what, "parallelism": "none"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": what + ", float64 NumPy"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_1m")
    ap.add_argument("--no-prefill", action="store_true", help="skip the csa_prefill_128k layer")
    ap.add_argument("--no-256k", action="store_true", help="skip the decode_256k run")
    ap.add_argument("--no-fp8kv", action="store_true", help="skip the decode_1m run with FP8 KV caches")
    ap.add_argument("--prefill-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the decode step eagerly")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world, rank, local = dist_setup() if torch.cuda.is_available() else (1, 0, 0)
    if args.impl == "reference":
        run_reference(args, world, rank)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)
    wl = synth.WORKLOADS[args.workload]
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    main_run = decode_run(wl, args, dev, stream, world, rank, want_cpu)
    extra = None
    if not args.no_256k and args.workload != "decode_256k":
        extra = decode_run(synth.WORKLOADS["decode_256k"], args, dev, stream, world, rank, False, e2e=False)
        extra["workload"] = "decode_256k"
    torch.cuda.empty_cache()
    fp8kv = None
    if not args.no_fp8kv and args.workload == "decode_1m":
        fp8kv = decode_run(synth.WORKLOADS["decode_1m_fp8kv"], args, dev, stream, world, rank, False, e2e=False)
        fp8kv["workload"] = "decode_1m_fp8kv"
    torch.cuda.empty_cache()
    prefill = None
    if not args.no_prefill:
        prefill = prefill_run(args, dev, stream, world, want_cpu)

    line = {
        "metric": METRIC, "value": main_run["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": main_run["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "global_batch": world * wl.B, "seq_len": wl.ctx,
                   "positions": main_run["positions"],
                   "layers": list(wl.layers), "heads": wl.H, "head_dim": wl.d, "top_k": wl.k,
                   "window": wl.w, "indexer_keys": "e4m3" if wl.fp8_keys else "bf16",
                   "parallelism": f"replicas{world}" if world > 1 else "none",
                   "launch": main_run["launch"], "l2": "flushed between timed steps",
                   "steps": "consecutive decode positions; CSA blocks complete every 4th step, "
                            "one HCA block mid-run"},
        "roofline": main_run["roofline"],
        "step_hbm": main_run["step_hbm"],
        "ms_per_step_by_kind": main_run["ms_per_step_by_kind"],
        "clocks": main_run["clocks"],
        "e2e": main_run.get("e2e"),
        "gpu_launches": main_run["gpu_launches"],
        "kernels_ms_per_step": main_run["kernels_ms_per_step"],
        "cpu_baseline": main_run.get("cpu_baseline"),
        "decode_256k": extra,
        "decode_1m_fp8kv": fp8kv,
        "prefill": prefill,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier(world)
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
