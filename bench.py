#!/usr/bin/env python
"""Benchmark: DiffQKV decode attention KV-cache bandwidth at 32k context vs GQA.

One step = one diffqkv_decode call over the whole batch of the Sigma-1.5B-shaped
decode workload (B=16, n_q=16, n_k=4, n_v=16, d_k=64, d_v=128, 32768 cached
positions per sequence, bf16 N(0,1) inputs, seed 1): head mapping, split
scores, online-softmax partials, split P.V, combine -- one kernel launch.
The symmetric GQA control (n_k=n_v=16, d_k=d_v=128, same seed) is timed the
same way and reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, one process per GPU; every rank decodes its own
full batch (independent sequences: weak scaling, no collective on the data
path); the time is the max over ranks.  ``--impl reference`` times the fp64
CPU oracle on a bounded sample of the same workload (rank 0 only).
Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "decode attn KV-cache GB/s (% of HBM peak) and us/step at 32k ctx vs GQA"
UNIT = "GB/s"
WORKLOAD = wl.DECODE_32K
CONTROL = wl.DECODE_32K_GQA
PROFILE = os.path.join(ROOT, "profiles", "decode_split_combine_b16_t32768.md")
KERNEL_SOURCES = ["asymmetric_head_kv_b200/csrc/decode.cu", "asymmetric_head_kv_b200/csrc/common.cuh",
                  "asymmetric_head_kv_b200/csrc/api.cu"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}

# Reduced cases for ncu captures: inputs larger than L2 (126 MB), a few GB at most.
PROFILE_CASES = {
    "decode_b4_t32768": wl.DecodeWorkload("decode_b4_t32768", wl.DIFFQKV, 4, 32768, seed=1),
    "decode_gqa_b4_t32768": wl.DecodeWorkload("decode_gqa_b4_t32768", wl.GQA_CONTROL, 4, 32768, seed=1),
    "prefill_b2_s8192": wl.PREFILL_8K,
    "prefill_gqa_b2_s8192": wl.PREFILL_8K_GQA,
    "topv_b4_t65536": wl.TOPV_64K,
    "decode_paged_b4_t32768_p16": wl.DecodeWorkload("decode_paged_b4_t32768_p16", wl.DIFFQKV, 4, 32768, seed=1,
                                                    page_size=16),
    "decode_b1_t512": wl.DECODE_SMALL,
    "augq_t16384": wl.AUGQ_16K,
}
L2_FLUSH_BYTES = 256 << 20  # written between timed calls whose inputs fit in the 126 MB L2


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--e2e-steps", type=int, default=5)
    p.add_argument("--profile-case", choices=sorted(PROFILE_CASES), default=None,
                   help="run a few launches of one kernel on a reduced case for ncu; prints no bench line")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this kernel source."""
    if not os.path.exists(PROFILE):
        return None
    text = open(PROFILE).read()
    m_hash = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", text)
    m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_tr or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_tr.group(1))


def _clock_sampler_proc(device_index: int, conn, period_s: float):
    """Child process: samples the SM clock and the clock-event reasons through NVML (read-only) until
    told to stop, then sends back (timestamp, MHz, reason mask) samples.  A separate process, so the
    samples keep coming while the parent waits on the GPU."""
    try:
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
        max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
    except Exception:  # no NVML: no samples
        conn.send((None, []))
        return
    conn.send(("ready", max_mhz))
    samples = []
    while not conn.poll():
        try:
            samples.append((time.monotonic(), pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                            pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)))
        except Exception:
            pass
        time.sleep(period_s)
    conn.recv()
    conn.send((max_mhz, samples))


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML during the timed region, in a child
    process started before the warm-up; only the samples taken between entering and leaving the
    context count."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.0002):
        import multiprocessing as mp
        ctx = mp.get_context("spawn")
        self.conn, child = ctx.Pipe()
        self.proc = ctx.Process(target=_clock_sampler_proc, args=(device_index, child, period_s), daemon=True)
        self.proc.start()
        first = self.conn.recv()
        self.ok = first[0] == "ready"
        self.max_mhz = first[1] if self.ok else None
        self.samples, self.reasons = [], set()
        self.t0 = self.t1 = None

    def __enter__(self):
        self.t0 = time.monotonic()
        return self

    def __exit__(self, *a):
        self.t1 = time.monotonic()
        return False

    def close(self):
        if self.ok:
            self.conn.send("stop")
            _, samples = self.conn.recv()
            for t, mhz, mask in samples:
                if self.t0 is not None and self.t0 <= t <= self.t1:
                    self.samples.append(mhz)
                    for name, bit in self.REASONS.items():
                        if mask & bit and name != "gpu_idle":
                            self.reasons.add(name)
        self.proc.join(timeout=10)

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank scalar (device time) over all ranks."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(bytes_per_rank: int, world: int, region_ms_max: float, steps: int) -> float:
    """Whole-job GB/s: bytes every rank moved in one step, over the slowest rank's time per step."""
    return bytes_per_rank * world / (region_ms_max / steps * 1e-3) / 1e9


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def time_decode(ak, w: wl.DecodeWorkload, steps: int, warmup: int, world: int, sampler=None):
    """Times `steps` decode calls; returns dict with region time, per-launch times, bytes."""
    dev = torch.device("cuda", torch.cuda.current_device())
    d = wl.make_decode_inputs(w, dev)
    out = torch.empty((w.batch, w.shape.n_q, w.shape.d_v), dtype=torch.bfloat16, device=dev)
    ws = ak.decode_workspace(d["q"], d["k_cache"], d["v_cache"])
    msl = int(d["seq_lens"].max())
    stream = torch.cuda.current_stream()

    def step():
        ak.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], scale=d["scale"], max_seq_len=msl,
                  out=out, workspace=ws, stream=stream)

    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize()
    assert ak.workspace_status(ws) == 0
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        for i in range(steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        # wait for the last step without holding the interpreter lock the whole time
        while not ends[-1].query():
            time.sleep(0.0001)
        torch.cuda.synchronize()
    barrier(world)
    region_ms = starts[0].elapsed_time(ends[-1])
    per_launch = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    nbytes = wl.decode_kv_bytes(w.shape, d["seq_lens"].cpu())
    res = {"region_ms": region_ms, "launch_ms_mean": statistics.fmean(per_launch),
           "launch_ms_median": statistics.median(per_launch), "kv_bytes": nbytes, "inputs": d, "out": out}
    return res


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def time_e2e(ak, w: wl.DecodeWorkload, d_dev: dict, steps: int):
    """Same step through the host-buffer C-ABI entry point: H2D of all inputs, decode, D2H of the output."""
    host = {k: d_dev[k].cpu().pin_memory() for k in ("q", "k_cache", "v_cache", "seq_lens")}
    out_host = torch.empty((w.batch, w.shape.n_q, w.shape.d_v), dtype=torch.bfloat16).pin_memory()
    dev = {k: torch.empty_like(d_dev[k]) for k in ("q", "k_cache", "v_cache", "seq_lens")}
    dev["out"] = torch.empty((w.batch, w.shape.n_q, w.shape.d_v), dtype=torch.bfloat16, device=d_dev["q"].device)
    dev["workspace"] = ak.decode_workspace(d_dev["q"], d_dev["k_cache"], d_dev["v_cache"])
    msl = int(host["seq_lens"].max())
    stream = torch.cuda.current_stream()

    def step():
        ak.decode_from_host(host["q"], host["k_cache"], host["v_cache"], host["seq_lens"], out_host, dev,
                            scale=w.shape.scale, max_seq_len=msl, stream=stream)

    step()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        step()
    e.record(stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    h2d = sum(host[k].numel() * host[k].element_size() for k in host)
    d2h = out_host.numel() * out_host.element_size()
    return ms, h2d, d2h


def oracle_sample_rate(w: wl.DecodeWorkload, d_cpu: dict, budget_s: float):
    """fp64 oracle on a bounded sample of (b, h) rows; GB/s attributed pro rata to the step's KV bytes."""
    import oracle

    rows_total = w.batch * w.shape.n_q
    step_bytes = wl.decode_kv_bytes(w.shape, d_cpu["seq_lens"])
    threads = os.cpu_count() or 1
    # calibrate on one row per thread, then size the sample to the budget
    n = min(rows_total, threads)
    rows = [(i // w.shape.n_q, i % w.shape.n_q) for i in range(n)]
    t0 = time.perf_counter()
    oracle.decode(d_cpu["q"], d_cpu["k_cache"], d_cpu["v_cache"], d_cpu["seq_lens"], d_cpu["scale"], rows=rows,
                  threads=threads)
    dt = time.perf_counter() - t0
    n = int(max(1, min(rows_total, n * budget_s / max(dt, 1e-6))))
    rows = [(i // w.shape.n_q, i % w.shape.n_q) for i in range(n)]
    t0 = time.perf_counter()
    oracle.decode(d_cpu["q"], d_cpu["k_cache"], d_cpu["v_cache"], d_cpu["seq_lens"], d_cpu["scale"], rows=rows,
                  threads=threads)
    dt = time.perf_counter() - t0
    nbytes = step_bytes * n / rows_total
    return {"value": nbytes / dt / 1e9, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n} of {rows_total} (b, h) rows of one step ({n / rows_total:.0%} of its KV bytes), "
                      f"fp64 C oracle, {dt:.2f} s", "seconds": dt}


def bench_config(world: int) -> dict:
    """The workload both arms (the kernels and the oracle) measure, under the same keys."""
    s = WORKLOAD.shape
    return {"workload": WORKLOAD.name, "batch_per_gpu": WORKLOAD.batch, "context": WORKLOAD.t_max,
            "n_q": s.n_q, "n_k": s.n_k, "n_v": s.n_v, "d_k": s.d_k, "d_v": s.d_v,
            "parallelism": f"replicas x{world}",
            "l2": "inputs (2.42 GB) larger than L2 (126 MB); no flush",
            "kv_bytes_per_gpu_step": wl.decode_kv_bytes(s, WORKLOAD.seq_lens())}


def run_reference(args, world, rank):
    if rank != 0:
        return
    budget = max(0.5, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    d = wl.make_decode_inputs(WORKLOAD, "cpu")
    total_bytes, total_s, info = 0.0, 0.0, None
    for i in range(args.warmup + args.steps):
        info = oracle_sample_rate(WORKLOAD, d, budget)
        if i >= args.warmup:
            total_bytes += info["value"] * 1e9 * info["seconds"]
            total_s += info["seconds"]
    value = total_bytes / total_s / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": info["cores"], "kind": "oracle",
                         "sample": info["sample"] + " per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile_case(name: str, launches: int = 4):
    import asymmetric_head_kv_b200 as ak

    w = PROFILE_CASES[name]
    dev = torch.device("cuda", 0)
    if isinstance(w, wl.AugQWorkload):
        d = wl.make_augq_inputs(w, dev)
        for _ in range(launches):
            ak.augq_project(d["x"], d["w_gate"], d["w_up"], d["w_down"])
        what = f"flops/call {wl.augq_flops(w)} (two launches per call)"
    elif isinstance(w, wl.PrefillWorkload):
        d = wl.make_prefill_inputs(w, dev)
        out = torch.empty((w.batch, w.seq, w.shape.n_q, w.shape.d_v), dtype=torch.bfloat16, device=dev)
        for _ in range(launches):
            ak.prefill_causal(d["q"], d["k"], d["v"], scale=d["scale"], out=out)
        what = f"causal flops/launch {wl.prefill_causal_flops(w.shape, w.batch, w.seq)}"
    elif w.page_size:
        d = wl.random_paged_inputs(w.batch, w.t_max // w.page_size + 1, w.page_size, w.shape, seed=w.seed,
                                   seq_lens=[w.t_max] * w.batch, device=dev)
        for _ in range(launches):
            ak.decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"],
                            scale=d["scale"], max_seq_len=w.t_max)
        what = f"kv bytes/launch {wl.decode_kv_bytes(w.shape, d['seq_lens'].cpu())}"
    elif w.topk:
        d = wl.make_decode_inputs(w, dev)
        for _ in range(launches):
            ak.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], w.topk, scale=d["scale"])
        what = f"algorithmic bytes/launch {topv_bytes(w, d['seq_lens'])}"
    else:
        d = wl.make_decode_inputs(w, dev)
        ws = ak.decode_workspace(d["q"], d["k_cache"], d["v_cache"])
        for _ in range(launches):
            ak.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], scale=d["scale"], workspace=ws)
        what = f"kv bytes/launch {wl.decode_kv_bytes(w.shape, d['seq_lens'])}"
        assert ak.workspace_status(ws) == 0
    torch.cuda.synchronize()
    assert ak.device_status() == 0
    print(f"profile case {name}: {launches} launches, {what}")


def topv_bytes(w: wl.DecodeWorkload, seq_lens) -> int:
    """Selective-V algorithmic bytes: every cached K row once, plus the selected V rows."""
    lens = torch.as_tensor(seq_lens, dtype=torch.int64).clamp(min=0)
    k_bytes = int(lens.sum()) * w.shape.n_k * w.shape.d_k * 2
    v_rows = int(lens.clamp(max=w.topk).sum()) * w.shape.n_q
    return k_bytes + v_rows * w.shape.d_v * 2


PATHS_TIMING = ("per-call CUDA events on the launch stream, median of the steps; before each call (untimed) a "
                "256 MB buffer is written (L2 flush) and then read, so the call finds none of its inputs in L2 and "
                "does not pay for the write-back of the flush's dirty lines")


def _timed_calls(fn, steps: int, flush: torch.Tensor):
    """Per-call CUDA-event times (ms) on the current stream.  Before every call, untimed: the flush
    buffer (larger than L2) is written, which evicts the call's inputs, then read, so the dirty lines
    the write left behind are written back before the call starts instead of during it."""
    stream = torch.cuda.current_stream()
    times = []
    for _ in range(steps):
        flush.add_(1)
        flush.sum()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        fn()
        e.record(stream)
        times.append((s, e))
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in times]


def time_paths(ak, peaks, steps: int, warmup: int):
    """Causal prefill (tensor cores) and selective-V decode, one call = one step of each."""
    dev = torch.device("cuda", torch.cuda.current_device())
    flush = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    res = {}
    bf16_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    for w in (wl.PREFILL_8K, wl.PREFILL_8K_GQA):
        d = wl.make_prefill_inputs(w, dev)
        out = torch.empty((w.batch, w.seq, w.shape.n_q, w.shape.d_v), dtype=torch.bfloat16, device=dev)
        fn = lambda: ak.prefill_causal(d["q"], d["k"], d["v"], scale=d["scale"], out=out)  # noqa: E731
        for _ in range(max(3, warmup)):
            fn()
        ms = statistics.median(_timed_calls(fn, steps, flush))
        flops = wl.prefill_causal_flops(w.shape, w.batch, w.seq)
        tf = flops / (ms * 1e-3) / 1e12
        res[w.name] = {"ms": ms, "causal_flops": flops, "tflops": tf, "bound": "tensor", "peak_tflops": bf16_peak,
                       "frac": tf / bf16_peak, "frac_kind": "FLOP-derived tensor fraction (causal FLOPs / event "
                       "time / peak)", "peak_source": "bf16_tflops (burst, cuBLAS bf16 GEMM)"}
        del d, out
    # chunked prefill: 2048 new rows over an 8192-position prefix (batch 2, DiffQKV shape)
    P, S, w = 8192, 2048, wl.PREFILL_8K
    d = wl.random_prefill_inputs(w.batch, P + S, w.shape, seed=w.seed, device=dev)
    qn = d["q"][:, P:].contiguous()
    out = torch.empty((w.batch, S, w.shape.n_q, w.shape.d_v), dtype=torch.bfloat16, device=dev)
    fn = lambda: ak.prefill_causal_prefix(qn, d["k"], d["v"], P, scale=d["scale"], out=out)  # noqa: E731
    for _ in range(max(3, warmup)):
        fn()
    ms = statistics.median(_timed_calls(fn, steps, flush))
    flops = 2 * w.batch * w.shape.n_q * (S * P + S * (S + 1) // 2) * (w.shape.d_k + w.shape.d_v)
    tf = flops / (ms * 1e-3) / 1e12
    res["prefill_prefix_b2_p8192_s2048"] = {"ms": ms, "causal_flops": flops, "tflops": tf, "bound": "tensor",
                                            "peak_tflops": bf16_peak, "frac": tf / bf16_peak,
                                            "frac_kind": "FLOP-derived tensor fraction",
                                            "peak_source": "bf16_tflops (burst, cuBLAS bf16 GEMM)"}
    # the same chunked prefill with K and V in 16-position pages dealt out in random order
    page = 16
    per_seq = (P + S + page - 1) // page
    g = torch.Generator().manual_seed(w.seed + 7)
    perm = torch.randperm(w.batch * per_seq, generator=g).to(torch.int32).view(w.batch, per_seq)
    table = perm.to(dev).contiguous()
    kp = torch.empty((w.batch * per_seq, page, w.shape.n_k, w.shape.d_k), dtype=torch.bfloat16, device=dev)
    vp = torch.empty((w.batch * per_seq, page, w.shape.n_v, w.shape.d_v), dtype=torch.bfloat16, device=dev)
    kp[table.long().view(-1)] = d["k"].view(w.batch * per_seq, page, w.shape.n_k, w.shape.d_k)
    vp[table.long().view(-1)] = d["v"].view(w.batch * per_seq, page, w.shape.n_v, w.shape.d_v)
    fn = lambda: ak.prefill_causal_paged(qn, kp, vp, table, P, scale=d["scale"], out=out)  # noqa: E731
    for _ in range(max(3, warmup)):
        fn()
    ms = statistics.median(_timed_calls(fn, steps, flush))
    tf = flops / (ms * 1e-3) / 1e12
    res["prefill_prefix_paged_b2_p8192_s2048_page16"] = {
        "ms": ms, "causal_flops": flops, "tflops": tf, "bound": "tensor", "peak_tflops": bf16_peak,
        "frac": tf / bf16_peak, "frac_kind": "FLOP-derived tensor fraction",
        "peak_source": "bf16_tflops (burst, cuBLAS bf16 GEMM)"}
    assert ak.device_status() == 0
    del d, qn, out, kp, vp, table

    # the small decode case (batch 1, 512 positions: 2.36 MB, launch/latency bound): microseconds
    # per call with L2 flushed before each call
    w = wl.DECODE_SMALL
    d = wl.make_decode_inputs(w, dev)
    ws_s = ak.decode_workspace(d["q"], d["k_cache"], d["v_cache"])
    out_s = torch.empty((w.batch, w.shape.n_q, w.shape.d_v), dtype=torch.bfloat16, device=dev)
    fn = lambda: ak.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], scale=d["scale"],  # noqa: E731
                           out=out_s, workspace=ws_s)
    for _ in range(max(3, warmup)):
        fn()
    ms = statistics.median(_timed_calls(fn, max(20, steps), flush))
    nbytes = wl.decode_kv_bytes(w.shape, d["seq_lens"].cpu())
    res[w.name] = {"us": ms * 1e3, "kv_bytes": nbytes, "gbs": nbytes / (ms * 1e-3) / 1e9,
                   "bound": "launch/latency (L2 flushed between calls)", "launches_per_call": 1}
    del d, ws_s, out_s

    # decode step with the KV-cache append fused in: 16 sequences of 32767 cached positions, the
    # new token goes to position 32767; bytes = the cached K/V read plus the new rows written
    w = WORKLOAD
    d = wl.make_decode_inputs(w, dev)
    lens = (d["seq_lens"] - 1).contiguous()
    g = torch.Generator(device=dev).manual_seed(w.seed + 100)
    k_new = torch.randn(w.batch, w.shape.n_k, w.shape.d_k, generator=g, device=dev).to(torch.bfloat16)
    v_new = torch.randn(w.batch, w.shape.n_v, w.shape.d_v, generator=g, device=dev).to(torch.bfloat16)
    ws_d = ak.decode_workspace(d["q"], d["k_cache"], d["v_cache"])
    out_d = torch.empty((w.batch, w.shape.n_q, w.shape.d_v), dtype=torch.bfloat16, device=dev)
    fn = lambda: ak.decode_append(d["q"], k_new, v_new, d["k_cache"], d["v_cache"], lens,  # noqa: E731
                                  scale=d["scale"], out=out_d, workspace=ws_d)
    for _ in range(max(3, warmup)):
        fn()
    ms = statistics.median(_timed_calls(fn, steps, flush))
    nbytes = wl.decode_kv_bytes(w.shape, lens.cpu()) + w.batch * w.shape.kv_elems_per_token * wl.BF16_BYTES
    hbm = float(peaks["hbm_gbs"])
    res["decode_append_b16_t32768"] = {"us": ms * 1e3, "algorithmic_bytes": nbytes,
                                       "gbs": nbytes / (ms * 1e-3) / 1e9, "bound": "hbm", "peak_gbs": hbm,
                                       "frac": nbytes / (ms * 1e-3) / 1e9 / hbm, "launches_per_call": 1}
    assert ak.workspace_status(ws_d) == 0 and ak.device_status() == 0
    del d, ws_d, out_d

    # the same 16 x 32768 decode over paged caches: K and V page pools with one block table, pages
    # dealt out to the sequences in random order
    for page_size in (16, 64):
        d = wl.random_paged_inputs(w.batch, w.t_max // page_size + 1, page_size, w.shape, seed=w.seed,
                                   seq_lens=[w.t_max] * w.batch, device=dev)
        ws_p = ak.decode_workspace(ak.make_dims(w.batch, w.shape.n_q, w.shape.n_k, w.shape.n_v, w.shape.d_k,
                                                w.shape.d_v, w.shape.scale), device=dev)
        out_p = torch.empty((w.batch, w.shape.n_q, w.shape.d_v), dtype=torch.bfloat16, device=dev)
        fn = lambda: ak.decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"],  # noqa: E731
                                     d["seq_lens"], scale=d["scale"], max_seq_len=w.t_max, out=out_p,
                                     workspace=ws_p)
        for _ in range(max(3, warmup)):
            fn()
        ms = statistics.median(_timed_calls(fn, steps, flush))
        nbytes = wl.decode_kv_bytes(w.shape, d["seq_lens"].cpu())
        res[f"decode_paged_b16_t32768_p{page_size}"] = {
            "us": ms * 1e3, "kv_bytes": nbytes, "gbs": nbytes / (ms * 1e-3) / 1e9, "bound": "hbm",
            "peak_gbs": hbm, "frac": nbytes / (ms * 1e-3) / 1e9 / hbm, "launches_per_call": 1}
        assert ak.workspace_status(ws_p) == 0
        del d, ws_p, out_p

    # query fold for d_q != d_k (the K up-projection moved onto the query): 16 decode rows of 16 query
    # heads, d_q = 192 (an augmented query of 3072 over 16 heads) onto d_k = 64; launch/latency bound
    B, s_, d_q = 16, wl.DIFFQKV, 192
    g = torch.Generator(device=dev).manual_seed(5)
    q_aug = torch.randn(B, s_.n_q, d_q, generator=g, device=dev).to(torch.bfloat16)
    w_up = (torch.randn(s_.n_k, d_q, s_.d_k, generator=g, device=dev) / 8).to(torch.bfloat16)
    q_fold = torch.empty((B, s_.n_q, s_.d_k), dtype=torch.bfloat16, device=dev)
    fn = lambda: ak.fold_query(q_aug, w_up, n_k=s_.n_k, out=q_fold)  # noqa: E731
    for _ in range(max(3, warmup)):
        fn()
    ms = statistics.median(_timed_calls(fn, max(20, steps), flush))
    nbytes = (q_aug.numel() + w_up.numel() + q_fold.numel()) * 2
    res["fold_query_b16_dq192_dk64"] = {"us": ms * 1e3, "bytes": nbytes, "gbs": nbytes / (ms * 1e-3) / 1e9,
                                        "bound": "launch/latency (L2 flushed between calls)",
                                        "launches_per_call": 1}
    del q_aug, w_up, q_fold

    # augmented query projection of Sigma-1.5B's attention (hidden 2048 -> gated 3072 -> 2048 query
    # features) for the 16384 rows of the 2 x 8192 prefill: two tcgen05 GEMMs, TFLOP/s
    w = wl.AUGQ_16K
    d = wl.make_augq_inputs(w, dev)
    h_a = torch.empty((w.tokens, w.d_inter), dtype=torch.bfloat16, device=dev)
    q_a = torch.empty((w.tokens, w.d_out), dtype=torch.bfloat16, device=dev)
    fn = lambda: ak.augq_project(d["x"], d["w_gate"], d["w_up"], d["w_down"], h_out=h_a, q_out=q_a)  # noqa: E731
    for _ in range(max(3, warmup)):
        fn()
    ms = statistics.median(_timed_calls(fn, steps, flush))
    flops = wl.augq_flops(w)
    tf = flops / (ms * 1e-3) / 1e12
    res[w.name] = {"us": ms * 1e3, "flops": flops, "tflops": tf, "bound": "tensor", "peak_tflops": bf16_peak,
                   "frac": tf / bf16_peak, "frac_kind": "FLOP-derived (2 GEMMs' FLOPs / event time / peak)",
                   "peak_source": "bf16_tflops (burst, cuBLAS bf16 GEMM)", "launches_per_call": 2}
    assert ak.device_status() == 0
    del d, h_a, q_a

    w = wl.TOPV_64K
    d = wl.make_decode_inputs(w, dev)
    ws = ak.decode_topv_workspace(ak.make_dims(w.batch, w.shape.n_q, w.shape.n_k, w.shape.n_v, w.shape.d_k,
                                               w.shape.d_v, w.shape.scale), w.t_max, w.topk, dev)
    fn = lambda: ak.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], w.topk,  # noqa: E731
                                scale=d["scale"], workspace=ws)
    for _ in range(max(3, warmup)):
        fn()
    ms = statistics.median(_timed_calls(fn, steps, flush))
    nbytes = topv_bytes(w, d["seq_lens"].cpu())
    hbm = float(peaks["hbm_gbs"])
    res[w.name] = {"us": ms * 1e3, "algorithmic_bytes": nbytes, "gbs": nbytes / (ms * 1e-3) / 1e9,
                   "bound": "hbm", "peak_gbs": hbm, "frac": nbytes / (ms * 1e-3) / 1e9 / hbm,
                   "launches_per_call": 1}
    # the same selection over paged caches (16-position pages dealt out in random order)
    del d
    dp = wl.random_paged_inputs(w.batch, w.t_max // 16 + 1, 16, w.shape, seed=w.seed, seq_lens=[w.t_max] * w.batch,
                                device=dev)
    ws_pg = ak.decode_topv_workspace(ak.make_dims(w.batch, w.shape.n_q, w.shape.n_k, w.shape.n_v, w.shape.d_k,
                                                  w.shape.d_v, w.shape.scale), (w.t_max // 16 + 1) * 16, w.topk, dev)
    fn = lambda: ak.decode_topv_paged(dp["q"], dp["k_pages"], dp["v_pages"], dp["block_table"],  # noqa: E731
                                      dp["seq_lens"], w.topk, scale=dp["scale"], workspace=ws_pg)
    for _ in range(max(3, warmup)):
        fn()
    ms = statistics.median(_timed_calls(fn, steps, flush))
    res[w.name + "_paged_p16"] = {"us": ms * 1e3, "algorithmic_bytes": nbytes, "gbs": nbytes / (ms * 1e-3) / 1e9,
                                  "bound": "hbm", "peak_gbs": hbm, "frac": nbytes / (ms * 1e-3) / 1e9 / hbm,
                                  "launches_per_call": 1}
    assert ak.workspace_status(ws_pg) == 0
    del dp, ws_pg
    d = wl.make_decode_inputs(w, dev)
    # the same selection with the pages' full-softmax weights (no renormalisation over the kept set)
    fn = lambda: ak.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], w.topk,  # noqa: E731
                                scale=d["scale"], workspace=ws, full_weights=True)
    for _ in range(max(3, warmup)):
        fn()
    ms = statistics.median(_timed_calls(fn, steps, flush))
    res[w.name + "_full_weights"] = {"us": ms * 1e3, "algorithmic_bytes": nbytes,
                                     "gbs": nbytes / (ms * 1e-3) / 1e9, "bound": "hbm", "peak_gbs": hbm,
                                     "frac": nbytes / (ms * 1e-3) / 1e9 / hbm, "launches_per_call": 1}
    assert ak.workspace_status(ws) == 0
    return res


def main():
    args = parse()
    if args.profile_case:
        run_profile_case(args.profile_case)
        return
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    import asymmetric_head_kv_b200 as ak

    torch.cuda.set_device(local)
    peaks, peak_src = load_peaks()
    sampler = ClockSampler(local)  # started before the first GPU work (a spawned process)
    main_res = time_decode(ak, WORKLOAD, args.steps, args.warmup, world, sampler)
    region_ms = max_over_ranks(main_res["region_ms"], world)
    ms_per_step = region_ms / args.steps
    total_bytes = main_res["kv_bytes"] * world
    value = weak_scaling_value(main_res["kv_bytes"], world, region_ms, args.steps)

    launch_ms = main_res["launch_ms_mean"]
    achieved = main_res["kv_bytes"] / (launch_ms * 1e-3) / 1e9
    peak = float(peaks["hbm_gbs"])
    traffic = profiled_traffic()
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": traffic, "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)",
                "kernel": "decode_split_combine_kernel", "launch_us_mean": launch_ms * 1e3,
                "launch_us_median": main_res["launch_ms_median"] * 1e3,
                "algorithmic_bytes_per_launch": main_res["kv_bytes"]}

    # symmetric GQA control, same seed and context
    ctrl = time_decode(ak, CONTROL, max(50, args.steps // 4), args.warmup, world)
    ctrl_ms = max_over_ranks(ctrl["region_ms"], world) / max(50, args.steps // 4)
    control = {"workload": CONTROL.name, "ms_per_step": ctrl_ms, "us_per_step": ctrl_ms * 1e3,
               "value": ctrl["kv_bytes"] * world / (ctrl_ms * 1e-3) / 1e9, "unit": UNIT,
               "kv_bytes_per_gpu": ctrl["kv_bytes"],
               "frac_of_peak": ctrl["kv_bytes"] / (ctrl["launch_ms_mean"] * 1e-3) / 1e9 / peak,
               "diffqkv_time_reduction": 1.0 - ms_per_step / ctrl_ms}
    del ctrl

    # long-context ragged decode (lengths 16384..131072) and its GQA control: the same kernel, per-launch events
    long_ctx = {}
    for w in (wl.DECODE_RAGGED, wl.DECODE_RAGGED_GQA):
        r = time_decode(ak, w, 50, args.warmup, world)
        gbs = r["kv_bytes"] / (r["launch_ms_mean"] * 1e-3) / 1e9
        long_ctx[w.name] = {"us_per_step": r["launch_ms_mean"] * 1e3, "kv_bytes": r["kv_bytes"], "gbs": gbs,
                            "frac_of_peak": gbs / peak, "steps": 50}
        del r
    rag, rag_gqa = long_ctx[wl.DECODE_RAGGED.name], long_ctx[wl.DECODE_RAGGED_GQA.name]
    long_ctx["diffqkv_time_reduction"] = 1.0 - rag["us_per_step"] / rag_gqa["us_per_step"]

    e2e_ms, h2d, d2h = time_e2e(ak, WORKLOAD, main_res["inputs"], args.e2e_steps)
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e = {"value": total_bytes / (e2e_ms * 1e-3) / 1e9, "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": args.e2e_steps,
           "api": "diffqkv_decode_from_host (pinned host buffers)"}

    sampler.close()
    paths = time_paths(ak, peaks, max(10, min(50, args.steps // 10)), args.warmup)

    cpu = None
    if rank == 0 and world == 1:
        d_cpu = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in main_res["inputs"].items()}
        info = oracle_sample_rate(WORKLOAD, d_cpu, 15.0)
        cpu = {k: info[k] for k in ("value", "unit", "cores", "kind", "sample")}
        del d_cpu

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "us_per_step": ms_per_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": bench_config(world),
            "pct_of_hbm_peak": 100.0 * achieved / peak,
            "gqa_control": control,
            "long_context": long_ctx,
            "paths": paths,
            "paths_timing": PATHS_TIMING,
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps,
            "clocks": sampler.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
