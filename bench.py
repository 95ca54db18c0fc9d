#!/usr/bin/env python
"""Throughput of the CSA + HCA compressed-attention hot path on B200.

One step = one decode step of the decode_1m workload through the C ABI:
4 sequences x 4 layers (CSA, HCA, CSA, HCA) at a cached context of 1,048,576
tokens (CSA 4:1 with e4m3 indexer keys and top-1024, HCA 128:1 dense, 128-token
window, 64 heads of 512 dims).  `value` = tokens/s over all ranks (each rank
runs its own 4 sequences: weak scaling, no collective on the data path).
With --prefill the line also carries the csa_prefill_128k layer (one CSA
prefill of 131,072 tokens: both compressors, indexer top-k, attention).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

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
    qo = 2 * H * d * 2
    return {
        "indexer_scores": B * (vc * key_row + HI * dI * 2 + HI * 4),
        "topk_rows": B * (vc * 4 + k * 4),
        "attn_decode_csa": B * ((k + w) * d * 2 + qo),
        "attn_decode_hca": B * ((vh + w) * d * 2 + qo),
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
        per += (J - 1) * 2 * wl.d * es + wl.d * es
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


def time_steps(step, K, stream, flush, world):
    """K steps, each bracketed by CUDA events on `stream`, L2 flushed between
    steps (outside the events).  Returns the max over ranks of the summed
    device time in ms."""
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(K):
            flush()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    total = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    return max_over_ranks(total, world)


# -------------------------------------------------------------- prefill ----

def prefill_layer_fn(wl, dev, stream):
    inp = synth.prefill_inputs(wl, dev)
    kvi, ik = inp["kv"], inp["ik"]
    q_pos = torch.arange(wl.n, device=dev, dtype=torch.int32)[None].repeat(wl.B, 1).contiguous()
    idx = torch.empty(wl.B, wl.n, wl.k, dtype=torch.int32, device=dev)
    out = torch.empty_like(inp["q"])

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
    return step


def prefill_flops(wl):
    n, m, k, w = wl.n, wl.m, wl.k, wl.w
    t = np.arange(n, dtype=np.int64)
    vis = (t + 1) // m
    pairs = int(vis.sum())
    keys = int(np.minimum(vis, k).sum() + np.minimum(w, t + 1).sum())
    idx_fl = pairs * wl.HI * wl.dI * 2
    att_fl = keys * wl.H * wl.d * 4
    return idx_fl, att_fl


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
        kv = npy(L["kv"][b])
        N_cap = kv.shape[0]
        if entry is not None and entry[0] < N_cap:
            kv[entry[0]] = entry[2]
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
    ap.add_argument("--prefill", action="store_true", help="also time csa_prefill_128k")
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
    layers = synth.decode_inputs(runtime.shard_workload(wl, rank), dev)
    io = runtime.StepIO(layers, dev)            # per-step inputs / outputs in one arena each
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    # the oracle's copy of the inputs, taken before any kernel runs
    layers_host = host_layers(layers) if want_cpu else None
    eager = runtime.DecodeStep(wl, layers, stream)
    step = eager
    launch_mode = "eager"
    if not args.no_graph:
        step = runtime.DecodeGraph(eager)
        launch_mode = "cuda_graph"
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.random_(0, 255)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    if api.device_error(stream) != 0:
        raise RuntimeError("device error flag set during warm-up")

    clocks = ClockSampler(local)
    clocks.start()
    total_ms = time_steps(step, args.steps, stream, flush, world)
    clk = clocks.stop()
    ms_per_step = total_ms / args.steps
    tokens = world * wl.B * args.steps
    value = tokens / (total_ms / 1000.0)

    # traced pass: per-kernel device time of the same K steps (eager launches,
    # so every kernel is bracketed by its own events)
    api.trace_enable(True)
    time_steps(eager, args.steps, stream, flush, world)
    traced = api.trace_collect()
    api.trace_enable(False)

    pk = peaks()
    per_bytes = decode_bytes_per_kernel(wl, wl.ctx)
    dom = max(traced.items(), key=lambda kv: kv[1][1])
    dname, (dl, dms) = dom
    key = kernel_bytes_key(dname)
    roof = None
    if key is not None:
        ach = per_bytes[key] / (dms / dl / 1000.0) / 1e9
        roof = {"kernel": dname, "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": ach / pk["hbm_gbs"], "traffic": ncu_traffic(dname),
                "peak_source": pk["source"], "launches": dl, "avg_us": 1000 * dms / dl}
    step_bytes = decode_step_bytes(wl, wl.ctx)
    step_frac = step_bytes / (ms_per_step / 1000.0) / 1e9 / pk["hbm_gbs"]

    # end to end: the step's inputs copied in from pinned host memory and its
    # outputs read back, one copy each way (the layers' tensors are views of
    # the two arenas)
    host_inp = io.inp.cpu().pin_memory()
    host_outp = torch.empty(io.out.shape, dtype=io.out.dtype).pin_memory()
    h2d = io.inp.numel()
    d2h = io.out.numel()

    def e2e_step():
        io.inp.copy_(host_inp, non_blocking=True)
        step()
        host_outp.copy_(io.out, non_blocking=True)

    with torch.cuda.stream(stream):
        e2e_step()
    torch.cuda.synchronize()
    e2e_ms = time_steps(e2e_step, args.steps, stream, flush, world)
    e2e_val = tokens / (e2e_ms / 1000.0)

    prefill = None
    if args.prefill:
        pw = synth.WORKLOADS["csa_prefill_128k"]
        pstep = prefill_layer_fn(pw, dev, stream)
        for _ in range(max(1, args.warmup // 3)):
            pstep()
        torch.cuda.synchronize()
        api.trace_enable(True)
        p_ms = time_steps(pstep, args.prefill_steps, stream, flush, world)
        ptr = api.trace_collect()
        api.trace_enable(False)
        idx_fl, att_fl = prefill_flops(pw)
        tot_fl = idx_fl + att_fl
        peak_tf = pk["bf16_tflops_sustained"]
        prefill = {"workload": pw.name, "tokens_per_s": world * pw.n * args.prefill_steps / (p_ms / 1000),
                   "ms_per_layer": p_ms / args.prefill_steps,
                   "tflops": tot_fl / (p_ms / args.prefill_steps / 1000) / 1e12,
                   "frac_of_bf16_peak": tot_fl / (p_ms / args.prefill_steps / 1000) / 1e12 / peak_tf,
                   "peak_tflops": peak_tf, "algorithmic_flops": tot_fl,
                   "kernels_ms_per_layer": {k_: v[1] / args.prefill_steps for k_, v in ptr.items()}}

    cpu = None
    if want_cpu:
        cpu = cpu_baseline(wl, layers_host)

    if api.device_error(stream) != 0:
        raise RuntimeError("device error flag set during the timed region")
    launches = sum(v[0] for v in traced.values()) // args.steps * args.steps
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "global_batch": world * wl.B, "seq_len": wl.ctx,
                   "layers": list(wl.layers), "heads": wl.H, "head_dim": wl.d, "top_k": wl.k,
                   "window": wl.w, "indexer_keys": "e4m3" if wl.fp8_keys else "bf16",
                   "parallelism": f"replicas{world}" if world > 1 else "none",
                   "launch": launch_mode, "l2": "flushed between timed steps"},
        "roofline": roof,
        "step_hbm": {"algorithmic_bytes": step_bytes, "frac": step_frac, "peak": pk["hbm_gbs"]},
        "clocks": clk,
        "e2e": {"value": e2e_val, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "kernels_ms_per_step": {k_: v[1] / args.steps for k_, v in traced.items()},
        "cpu_baseline": cpu,
        "prefill": prefill,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier(world)
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
