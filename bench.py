#!/usr/bin/env python3
"""Benchmark of the sparse MLA decode step (one JSON line on stdout).

One step = one decode call (smla_decode through the C ABI) over one batch of the
B=64, topk=512 workload (64 requests of 65536 tokens, 256 pages each, one
16384-page pool of 2.45 GB, 1% outlier rows).  Inputs rotate over 24 replicas
(distinct index sets and queries over the same pool, 24 x 23.3 MB = 560 MB
touched, more than 4x the 126 MB L2) so consecutive steps never find their KV
rows in L2.

The line also carries `per_config`: microseconds per call, algorithmic GB/s and the
roofline fraction of all five workloads of the sparse MLA decode target (B=1 topk=64;
B=1 topk=512; B=16 ragged; B=64; B=256), each timed on its own: B=64 and B=256 as
CUDA graphs over rotating replicas (more than 4x L2 per rotation), the three small
ones per call between L2 flushes (their whole page pools are at most 121 MB).

Modes:
  python bench.py [--gpus N] [--steps K] [--warmup W]      # CUDA path
  python bench.py --impl reference ...                     # the fp64 oracle on the host cores
Under torchrun (N > 1) each rank runs the same workload (its own seed) on its own
GPU with no data-path collective ("weak" scaling, replicas only); the step time
is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "sparse-MLA decode µs/call, queries·topk/s; HBM GB/s & TC TFLOP/s vs peak"
UNIT = "queries·topk/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CONFIG = 4
REPLICAS = 24
GRAPH_STEPS = 500


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(w, k=CONFIG):
    if k == 4:
        return (f"config4: B={w.B} H={w.H} topk={w.topk} seq_len=65536 (256 pages/request, "
                f"{w.num_pages}-page pool), e4m3 nope + UE8M0 per 64 + bf16 rope, 1% outlier rows x20, "
                f"sm_scale=512^-0.5")
    return (f"config{k}: {CONFIG_LABELS[k]}, {w.num_pages}-page pool, e4m3 nope + UE8M0 per 64 + bf16 rope, "
            f"sm_scale=512^-0.5")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        loaded = [r for r in rows if r["power"] > 1.2 * min(x["power"] for x in rows)] or rows
        reasons = []
        for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                          ("swp", "sw_power_cap")):
            if any(r[key].lower() == "active" for r in rows):
                reasons.append(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": rows[0]["smax"],
                "reasons": reasons, "samples": len(rows), "power_w_max": max(r["power"] for r in rows)}


def cpu_oracle_baseline(w, min_seconds: float, max_reps: int):
    """Time the fp64 oracle (as it stands) on full batches of the workload."""
    import oracle

    oracle.build()
    reps, t0 = 0, time.perf_counter()
    while True:
        r = reps % w.R
        oracle.decode(w.q[r], w.cache, w.block_table, w.topk_idx[r], w.seq_lens, w.sm_scale)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= max_reps:
            break
    units = reps * w.B * w.topk
    return {"value": units / el, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{reps} full batches of {w.B} queries x {w.topk} slots ({el:.1f} s, fp64, OpenMP)"}


def run_reference(args):
    """The oracle as the reference arm: K steps, each a bounded sample of (b, h) rows of the batch."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from sparse_mla_decode_fp8_b200 import workloads as W

    oracle.build()
    w = W.make_config(args.config, replicas=1)
    all_rows = np.array([(b, h) for b in range(w.B) for h in range(w.H)], np.int32)
    # calibrate: seconds per (b, h) row when a step holds one request's 64 rows
    t0 = time.perf_counter()
    oracle.decode(w.q[0], w.cache, w.block_table, w.topk_idx[0], w.seq_lens, w.sm_scale, rows=all_rows[:64])
    t_row = (time.perf_counter() - t0) / 64
    budget = 90.0
    per_step = int(max(1, min(len(all_rows), budget / max(1, args.steps) / max(t_row, 1e-6))))
    pos = 0

    def one_step():
        nonlocal pos
        sel = all_rows[np.arange(pos, pos + per_step) % len(all_rows)]
        pos = (pos + per_step) % len(all_rows)
        oracle.decode(w.q[0], w.cache, w.block_table, w.topk_idx[0], w.seq_lens, w.sm_scale, rows=sel)

    for _ in range(max(0, args.warmup)):
        one_step()
    t0 = time.perf_counter()
    for _ in range(max(1, args.steps)):
        one_step()
    el = time.perf_counter() - t0
    units = max(1, args.steps) * per_step * w.topk / w.H  # (query, slot) pairs: a row is one of 64 heads
    value = units / el
    sample = f"{per_step} (request, head) rows of the batch per step, fp64, OpenMP over requests"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": max(1, args.steps), "warmup": args.warmup, "ms_per_step": 1e3 * el / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(w, args.config), "B": w.B, "topk": w.topk, "H": w.H,
                       "parallelism": "host cores (OpenMP over requests)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


CONFIG_LABELS = {1: "B=1 topk=64 (launch-bound: a few us of work)", 2: "B=1 topk=512 (launch-bound: 4 CTAs)",
                 3: "B=16 topk=512, ragged seq_len in [256, 32768]", 4: "B=64 topk=512, seq_len 65536, 1% outliers",
                 5: "B=256 topk=512, seq_len in [1024, 8192], ~2M-token pool"}


def _config_entry(k, w, us, nsplit, timing, peaks):
    from sparse_mla_decode_fp8_b200 import workloads as W

    units = W.roofline_units(w.replica(0))
    t_hbm = units["bytes"] / (peaks["hbm_gbs"] * 1e9) * 1e6
    t_tc = units["flops"] / (peaks["bf16_tflops"] * 1e12) * 1e6
    gbs = units["bytes"] / (us * 1e-6) / 1e9
    return {"workload": CONFIG_LABELS[k], "B": w.B, "topk": w.topk, "nsplit": nsplit, "us_per_call": us,
            "algorithmic_bytes": units["bytes"], "gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
            "roofline_us": max(t_hbm, t_tc), "frac_of_roofline": max(t_hbm, t_tc) / us,
            "tc_tflops": units["flops"] / (us * 1e-6) / 1e12, "timing": timing}


def time_small_config(k, dev, peaks, calls: int = 40):
    """Per-call CUDA-event time of one small workload, 512 MB written between calls to flush L2."""
    import torch

    import sparse_mla_decode_fp8_b200 as smla
    from sparse_mla_decode_fp8_b200 import workloads as W

    w = W.make_config(k)
    q = torch.from_numpy(np.ascontiguousarray(w.q[0]).view(np.int16)).view(torch.bfloat16).to(dev)
    cache = torch.from_numpy(w.cache).to(dev)
    bt = torch.from_numpy(w.block_table).to(dev)
    idx = torch.from_numpy(np.ascontiguousarray(w.topk_idx[0])).to(dev)
    sl = torch.from_numpy(w.seq_lens).to(dev)
    nsplit = smla.num_splits(w.B, w.topk)
    ws = torch.zeros(smla.workspace_bytes(w.B, w.topk), dtype=torch.uint8, device=dev)
    out = torch.empty((w.B, 64, 512), dtype=torch.float32, device=dev)
    lse = torch.empty((w.B, 64), dtype=torch.float32, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(calls)]
    with torch.cuda.stream(stream):
        for _ in range(3):
            smla.decode(q, cache, bt, idx, sl, w.sm_scale, out=out, lse=lse, workspace=ws, stream=stream)
        for a, b in ev:
            flush.fill_(1)
            a.record(stream)
            smla.decode(q, cache, bt, idx, sl, w.sm_scale, out=out, lse=lse, workspace=ws, stream=stream)
            b.record(stream)
    stream.synchronize()
    assert smla.read_error(ws, stream) == 0
    us = statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3
    timing = f"median of {calls} calls, CUDA events around each, 512 MB written between calls (L2 flush)"
    return _config_entry(k, w, us, nsplit, timing, peaks)


def time_rotating_config(k, w, dev, peaks, calls: int = 200, reps: int = 5):
    """CUDA-graph time per call of a large workload over its rotating replicas."""
    import torch

    import sparse_mla_decode_fp8_b200 as smla

    cache = torch.from_numpy(w.cache).to(dev)
    bt = torch.from_numpy(w.block_table).to(dev)
    sl = torch.from_numpy(w.seq_lens).to(dev)
    qs = [torch.from_numpy(np.ascontiguousarray(w.q[r]).view(np.int16)).view(torch.bfloat16).to(dev)
          for r in range(w.R)]
    idxs = [torch.from_numpy(np.ascontiguousarray(w.topk_idx[r])).to(dev) for r in range(w.R)]
    nsplit = smla.num_splits(w.B, w.topk)
    ws = torch.zeros(smla.workspace_bytes(w.B, w.topk), dtype=torch.uint8, device=dev)
    out = torch.empty((w.B, 64, 512), dtype=torch.float32, device=dev)
    lse = torch.empty((w.B, 64), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(i):
        r = i % w.R
        smla.decode(qs[r], cache, bt, idxs[r], sl, w.sm_scale, out=out, lse=lse, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(3):
            step(i)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(calls):
            step(i)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g.replay()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    stream.synchronize()
    assert smla.read_error(ws, stream) == 0
    us = e0.elapsed_time(e1) * 1e3 / (calls * reps)
    from sparse_mla_decode_fp8_b200 import workloads as W

    per_rot = W.roofline_units(w.replica(0))["bytes"] * w.R
    timing = (f"CUDA graph of {calls} calls over {w.R} rotating replicas ({per_rot / 1e6:.0f} MB of KV+Q per "
              f"rotation > 4x L2), replayed {reps}x, CUDA events")
    del g
    return _config_entry(k, w, us, nsplit, timing, peaks)


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The largest of every rank's value (the job's time is its slowest rank's)."""
    if dist is None:
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, B: int, topk: int, steps: int, max_ms: float) -> float:
    """Whole-job (query, slot) pairs per second: every rank decodes B x topk per step."""
    return world * B * topk * steps / (max_ms * 1e-3)


def run_cuda(args):
    import torch

    import sparse_mla_decode_fp8_b200 as smla
    from sparse_mla_decode_fp8_b200 import build as smla_build
    from sparse_mla_decode_fp8_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    smla_build.build()
    smla.library()

    w = W.make_config(args.config, replicas=REPLICAS, seed=None if rank == 0 else 1000 + rank)
    B, topk, H = w.B, w.topk, w.H
    cache = torch.from_numpy(w.cache).to(dev)
    bt = torch.from_numpy(w.block_table).to(dev)
    sl = torch.from_numpy(w.seq_lens).to(dev)
    qs = [torch.from_numpy(np.ascontiguousarray(w.q[r]).view(np.int16)).view(torch.bfloat16).to(dev)
          for r in range(w.R)]
    idxs = [torch.from_numpy(np.ascontiguousarray(w.topk_idx[r])).to(dev) for r in range(w.R)]
    nsplit = smla.num_splits(B, topk)
    ws = torch.zeros(smla.workspace_bytes(B, topk), dtype=torch.uint8, device=dev)
    outs = [torch.empty((B, H, 512), dtype=torch.float32, device=dev) for _ in range(2)]
    lses = [torch.empty((B, H), dtype=torch.float32, device=dev) for _ in range(2)]
    stream = torch.cuda.Stream(device=dev)

    def step(i, s):
        r = i % w.R
        smla.decode(qs[r], cache, bt, idxs[r], sl, w.sm_scale, out=outs[i % 2], lse=lses[i % 2], workspace=ws,
                    stream=s)

    # warm-up (eager), then one graph of GRAPH_STEPS steps
    with torch.cuda.stream(stream):
        for i in range(max(3, args.warmup)):
            step(i, stream)
    stream.synchronize()
    assert smla.read_error(ws, stream) == 0
    gsteps = min(GRAPH_STEPS, args.steps)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(gsteps):
            step(i, stream)
    reps = max(1, (args.steps + gsteps - 1) // gsteps)
    steps = reps * gsteps
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    with ClockSampler(dev.index) as clk:
        with torch.cuda.stream(stream):
            # clocks under load before the timed region (graph replays for about a second)
            t_end = time.perf_counter() + 1.0
            while time.perf_counter() < t_end:
                g.replay()
                stream.synchronize()
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        stream.synchronize()
    barrier()
    elapsed_ms = e0.elapsed_time(e1)
    max_ms = max_over_ranks(elapsed_ms, dist, dev)
    assert smla.read_error(ws, stream) == 0

    # end to end through the public API: every step copies its inputs from pinned host memory to
    # the device, decodes, and copies O and LSE back to pinned host memory.  The copies run on
    # their own streams with two buffer sets, so step i+1's upload and step i-1's download overlap
    # step i's decode (as a serving loop would); every step still moves all of its bytes.
    e2e = None
    hq = [torch.from_numpy(np.ascontiguousarray(w.q[r]).view(np.int16)).view(torch.bfloat16).pin_memory()
          for r in range(w.R)]
    hidx = [torch.from_numpy(np.ascontiguousarray(w.topk_idx[r])).pin_memory() for r in range(w.R)]
    hbt = torch.from_numpy(w.block_table).pin_memory()
    hsl = torch.from_numpy(w.seq_lens).pin_memory()
    hout = [torch.empty((B, H, 512), dtype=torch.float32).pin_memory() for _ in range(2)]
    hlse = [torch.empty((B, H), dtype=torch.float32).pin_memory() for _ in range(2)]
    dq = [torch.empty_like(qs[0]) for _ in range(2)]
    didx = [torch.empty_like(idxs[0]) for _ in range(2)]
    dbt = [torch.empty_like(bt) for _ in range(2)]
    dsl = [torch.empty_like(sl) for _ in range(2)]
    up = torch.cuda.Stream(device=dev)
    down = torch.cuda.Stream(device=dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]
    e2e_steps = min(200, max(10, args.steps // 1000))

    def e2e_step(i):
        k, r = i % 2, i % w.R
        up.wait_event(ev_comp[k])  # the decode that last read buffer set k is done
        with torch.cuda.stream(up):
            dq[k].copy_(hq[r], non_blocking=True)
            didx[k].copy_(hidx[r], non_blocking=True)
            dbt[k].copy_(hbt, non_blocking=True)
            dsl[k].copy_(hsl, non_blocking=True)
        ev_up[k].record(up)
        stream.wait_event(ev_up[k])
        stream.wait_event(ev_down[k])  # output set k has been copied out
        smla.decode(dq[k], cache, dbt[k], didx[k], dsl[k], w.sm_scale, out=outs[k], lse=lses[k], workspace=ws,
                    stream=stream)
        ev_comp[k].record(stream)
        down.wait_event(ev_comp[k])
        with torch.cuda.stream(down):
            hout[k].copy_(outs[k], non_blocking=True)
            hlse[k].copy_(lses[k], non_blocking=True)
        ev_down[k].record(down)

    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier()
    a = torch.cuda.Event(enable_timing=True)
    b_ = torch.cuda.Event(enable_timing=True)
    a.record(up)
    for i in range(e2e_steps):
        e2e_step(i)
    b_.record(down)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(a.elapsed_time(b_), dist, dev)
    h2d = hq[0].numel() * 2 + hidx[0].numel() * 4 + hbt.numel() * 4 + hsl.numel() * 4
    d2h = hout[0].numel() * 4 + hlse[0].numel() * 4
    e2e = {"value": job_throughput(world, B, topk, e2e_steps, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": e2e_steps}

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    ms_step = max_ms / steps
    units = W.roofline_units(w.replica(0))
    peaks, peak_src = load_peaks()
    # a request in 2 splits merges inside the decode kernel (the CTA pair's fp32 adds): one launch
    # per call; 3 or more splits are merged by a second (combine) kernel
    launches_per_call = 1 if nsplit <= 2 else 2
    # this rank's own average duration of one decode launch over the timed region (graph replays on `stream`)
    call_ms = elapsed_ms / steps
    achieved_gbs = units["bytes"] / (call_ms * 1e-3) / 1e9
    achieved_tf = units["flops"] / (call_ms * 1e-3) / 1e12
    t_hbm_us = units["bytes"] / (peaks["hbm_gbs"] * 1e9) * 1e6
    t_tc_us = units["flops"] / (peaks["bf16_tflops"] * 1e12) * 1e6
    traffic = _profiled_traffic(args.config)
    line = {
        "metric": METRIC, "value": job_throughput(world, B, topk, steps, max_ms), "unit": UNIT, "n_gpus": world,
        "steps": steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step, "us_per_call": ms_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": workload_desc(w, args.config), "B": B, "topk": topk, "H": H, "nsplit": nsplit,
                   "l2": f"inputs larger than L2: {REPLICAS} rotating replicas, "
                         f"{REPLICAS * units['bytes'] / 1e6:.0f} MB of KV+Q touched per rotation > 126 MB",
                   "parallelism": f"replicas x{world} (no collective)", "timing": f"CUDA graph of {gsteps} steps "
                   f"replayed {reps}x, CUDA events, max over ranks"},
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved_gbs / peaks["hbm_gbs"], "traffic": traffic,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                     else "fallback 6.65 TB/s",
                     "kernel_us": call_ms * 1e3, "algorithmic_bytes": units["bytes"],
                     "roofline_us": max(t_hbm_us, t_tc_us), "frac_of_roofline": max(t_hbm_us, t_tc_us) / (call_ms * 1e3),
                     "tc_tflops": achieved_tf, "tc_peak_tflops": peaks["bf16_tflops"],
                     "tc_frac": achieved_tf / peaks["bf16_tflops"],
                     "per_launch": "CUDA events around the timed graph replays on the launching stream, "
                     f"divided by {steps} calls" + (" (decode + combine kernels)" if launches_per_call > 1 else
                                                    " (one decode kernel per call)")},
        "gpu_launches": steps * launches_per_call,
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    if not args.no_per_config and args.config == CONFIG:
        per = {}
        for k in (1, 2, 3):
            per[f"config{k}"] = time_small_config(k, dev, peaks)
        per["config4"] = _config_entry(4, w, call_ms * 1e3, nsplit, line["config"]["timing"] + " (the headline run)",
                                       peaks)
        w5 = W.make_config(5, replicas=8)
        per["config5"] = time_rotating_config(5, w5, dev, peaks)
        line["per_config"] = per
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_baseline(w, min_seconds=args.cpu_seconds, max_reps=200)
    print(json.dumps(line), flush=True)
    return 0


PROFILES = {4: "decode_kernel_B64_topk512.md", 5: "decode_kernel_B256_topk512.md"}


def _profiled_traffic(k: int):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this kernel source."""
    if k not in PROFILES:
        return None
    path = os.path.join(ROOT, "profiles", PROFILES[k])
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for ln in f:
            if ":" in ln and ln.split(":", 1)[0] in ("kernel_source_hash", "dram_bytes_per_launch"):
                k, v = ln.split(":", 1)
                fields[k] = v.strip()
    if fields.get("kernel_source_hash") != _kernel_hash() or "dram_bytes_per_launch" not in fields:
        return None
    return int(fields["dram_bytes_per_launch"])


def _code_tokens(src: str) -> str:
    """The source with its comments removed and whitespace collapsed: what the compiler sees."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def _kernel_hash() -> str:
    """Hash of the CUDA sources' code (comments and layout excluded), named in the ncu summaries."""
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_mla_decode_fp8_b200", "csrc")
    files = [os.path.join(csrc, name) for name in sorted(os.listdir(csrc))]
    for path in files + [os.path.join(ROOT, "include", "smla.h")]:
        with open(path, encoding="utf-8") as f:
            h.update(os.path.basename(path).encode() + b"\0" + _code_tokens(f.read()).encode() + b"\0")
    return h.hexdigest()[:16]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="time only the headline workload")
    ap.add_argument("--config", type=int, default=CONFIG, choices=[3, 4, 5],
                    help="workload of the timed run (default: the B=64 headline); 3 and 5 for profiling")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_cuda(args)


if __name__ == "__main__":
    sys.exit(main())
