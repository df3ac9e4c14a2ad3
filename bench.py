#!/usr/bin/env python
"""Benchmark of the B200 shifted-window attention forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {native,reference}]

One step = one alternating layer pair of the headline workload (the
Wan-like 720p video grid 21x45x80, 40 heads, d = 128, window 7x15x16, shifts
(0,0,0) then (3,7,8)): two launches of the fused kernel over inputs already
resident in HBM (3 x 774 MB, far larger than the 126 MB L2, so no flush is
needed between steps).  The metric is algorithmic TFLOP/s (4 * N * n_w * d *
heads per layer, summed over windows), also given as a fraction of the
measured B200 dense BF16 peak, with the speedup over the same kernel run as
full attention (window = whole grid).

With --gpus N > 1 the script runs under torchrun, one rank per GPU; the path
does not shard (every rank runs its own replica of the workload), so scaling
is weak and `value` is the FLOPs of all ranks over the slowest rank's time.

--impl reference times the fp64 CPU oracle instead (on rank 0 only), on
bounded samples of the same workload.

The last line printed on stdout by rank 0 is the JSON result.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "shifted-window attn fwd TFLOP/s & % of B200 BF16 peak; speedup vs full attn"
HEADLINE = "wan-720p-21x45x80-w7x15x16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_NAME = "swattn_fwd_pair_kernel"   # the head-dim-128 kernel the headline workload runs
KERNEL_SOURCES = ["shifted_window_attention_swattn_b200/csrc/swattn_sm100.cu",
                  "shifted_window_attention_swattn_b200/csrc/ptx_sm100.cuh",
                  "shifted_window_attention_swattn_b200/csrc/softmax_sm100.cuh"]


def strip_c_comments(text: str) -> str:
    """C/C++ source with its comments removed and runs of whitespace collapsed
    (string and character literals kept as they are), so that editing a comment
    does not change what the kernel hash identifies."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash(read=None) -> str:
    """Hash of the kernel sources, comments and whitespace aside.  `read(rel)`
    returns a file's text (default: the working tree)."""
    if read is None:
        def read(rel):
            with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
                return f.read()
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        h.update(strip_c_comments(read(rel)).encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            peaks = json.load(f)
        return peaks, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def load_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (key = value lines, '#' comments)."""
    path = os.path.join(ROOT, "profiles", "swattn_fwd_pair_kernel_wan720p_traffic.txt")
    rec = {}
    try:
        with open(path) as f:
            for line in f:
                line = line.strip()
                if line and not line.startswith("#") and "=" in line:
                    k, v = (x.strip() for x in line.split("=", 1))
                    rec[k] = v
    except OSError:
        return None
    if rec.get("kernel_source_hash") != kernel_source_hash():
        return None
    try:
        return {"dram_bytes_per_launch": float(rec["dram_bytes_per_launch"])}
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]), "util": float(parts[4]),
                             "reasons": {"hw_slowdown": parts[6], "hw_thermal_slowdown": parts[7],
                                         "sw_thermal_slowdown": parts[8], "sw_power_cap": parts[9]}})
            except ValueError:
                continue
        if not rows:
            return None
        loaded = [r for r in rows if r["util"] >= 50] or rows
        reasons = sorted({k for r in loaded for k, v in r["reasons"].items() if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(loaded)}


# ---------------------------------------------------------------- oracle timing (CPU)

def oracle_rows_sample(wl, q, k, v, n_rows, threads, seed):
    """Time the oracle's per-row path on n_rows random query rows of `wl`
    (alternating between the workload's shifts), split over `threads` host
    threads.  Returns (seconds, flops)."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(seed)
    jobs = []
    per = max(1, n_rows // (threads * len(wl.shifts)))
    for shift in wl.shifts:
        for _ in range(threads):
            tri = np.stack([rng.integers(0, wl.B, per), rng.integers(0, wl.N, per),
                            rng.integers(0, wl.heads, per)], axis=1).astype(np.int64)
            jobs.append((shift, tri))
    win_size_of_tok = {}
    for s in wl.shifts:
        tos, cnt = oracle.index_map(*wl.grid, wl.win, s)
        size = np.empty(wl.N, dtype=np.float64)
        for wid in range(tos.shape[0]):
            size[tos[wid, :cnt[wid]]] = cnt[wid]
        win_size_of_tok[s] = size
    flops = 0.0
    for shift, tri in jobs:
        flops += float((4.0 * win_size_of_tok[shift][tri[:, 1]] * wl.d).sum())
    qb, kb, vb = oracle._bits(q), oracle._bits(k), oracle._bits(v)

    def run(job):
        shift, tri = job
        oracle.swattn_rows(qb, kb, vb, wl.B, wl.heads, *wl.grid, wl.d, wl.win, shift, wl.scale, tri)

    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(run, jobs))
    return time.perf_counter() - t0, flops, per * len(jobs)


def host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ---------------------------------------------------------------- helpers

def wl_config(wl, extra=None):
    cfg = {"workload": wl.name, "B": wl.B, "heads": wl.heads, "d": wl.d,
           "grid_thw": list(wl.grid), "window_thw": list(wl.win),
           "shifts_thw": [list(s) for s in wl.shifts], "n_tokens": wl.N, "n_w": wl.n_w,
           "scale": "1/sqrt(d)", "step": "one layer per shift of the alternating pair",
           "l2": "inputs larger than L2 (no flush needed)"}
    if extra:
        cfg.update(extra)
    return cfg


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Maximum of a per-rank float over all ranks (identity on one rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, ms_max: float) -> float:
    """Throughput of the whole job: every rank's FLOPs over the slowest rank's time."""
    return flops_per_rank * world / (ms_max / 1e3) / 1e12


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ---------------------------------------------------------------- reference arm

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from shifted_window_attention_swattn_b200.inputs import BY_NAME, make_qkv
    wl = BY_NAME[args.workload]
    q, k, v = make_qkv(wl)
    threads = host_threads()
    # Size one step so that warmup + steps fit in about three minutes.
    t_probe, f_probe, _ = oracle_rows_sample(wl, q, k, v, threads * 2 * 4, threads, seed=1)
    rows_per_s = (threads * 2 * 4) / max(t_probe, 1e-6)
    budget_s = 150.0 / max(1, args.steps + args.warmup)
    n_rows = int(max(threads * len(wl.shifts), min(rows_per_s * budget_s, 200000)))
    for i in range(args.warmup):
        oracle_rows_sample(wl, q, k, v, n_rows, threads, seed=100 + i)
    tot_t, tot_f, rows_done = 0.0, 0.0, 0
    for i in range(args.steps):
        t, f, r = oracle_rows_sample(wl, q, k, v, n_rows, threads, seed=1000 + i)
        tot_t += t
        tot_f += f
        rows_done += r
    value = tot_f / tot_t / 1e12
    sample = (f"{rows_done // max(1, args.steps)} random query rows per step of {wl.name} "
              f"(both shifts), oracle per-row path (roll, window, fp64 softmax row, un-roll), "
              f"{threads} host threads, CPU {cpu_model()}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * tot_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": wl_config(wl),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- native arm

def time_launches(fn, iters, stream, flush=None):
    """Per-iteration CUDA-event timing on `stream`; optional L2 flush between
    iterations (outside the events).  Returns the list of ms."""
    import torch
    ms = []
    for _ in range(iters):
        if flush is not None:
            flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        ms.append(a.elapsed_time(b))
    return ms


def sweep_workloads(stream, flush, peak_tflops):
    """Per-workload table: windowed ms/layer per shift and full-attention ms,
    TFLOP/s, fraction of peak, speedup and its fraction of N/n_w."""
    import torch
    import shifted_window_attention_swattn_b200 as sw
    from shifted_window_attention_swattn_b200.inputs import WORKLOADS, make_qkv
    rows = []
    for wl in WORKLOADS:
        q, k, v = make_qkv(wl, device="cuda")
        out = torch.empty_like(q)
        f_win = sw.flops(wl.B, wl.heads, wl.grid, wl.d, wl.win)
        f_full = sw.flops(wl.B, wl.heads, wl.grid, wl.d, wl.grid)
        small = 3 * q.numel() * 2 < 2 * 126e6
        fl = flush if small else None
        per_shift = []
        for shift in wl.shifts:
            def fn(shift=shift):
                sw.swattn_fwd(q, k, v, wl.grid, wl.win, shift, wl.scale, out=out, stream=stream)
            time_launches(fn, 5, stream, fl)
            ms = statistics.median(time_launches(fn, 30, stream, fl))
            per_shift.append({"shift_thw": list(shift), "ms": ms,
                              "tflops": f_win / ms / 1e9, "frac_of_peak": f_win / ms / 1e9 / peak_tflops})

        def full():
            sw.swattn_fwd(q, k, v, wl.grid, wl.grid, (0, 0, 0), wl.scale, out=out, stream=stream)
        n_full = 3 if f_full > 1e13 else 10
        time_launches(full, 1, stream, fl)
        ms_full = statistics.median(time_launches(full, n_full, stream, fl))
        ms_win = statistics.mean(r["ms"] for r in per_shift)
        theo = f_full / f_win
        rows.append({"workload": wl.name, "flops_window": f_win, "flops_full": f_full,
                     "window": per_shift, "ms_window_mean": ms_win,
                     "ms_full": ms_full, "tflops_full": f_full / ms_full / 1e9,
                     "full_frac_of_peak": f_full / ms_full / 1e9 / peak_tflops,
                     "speedup_vs_full": ms_full / ms_win, "theoretical_speedup": theo,
                     "speedup_frac_of_theoretical": (ms_full / ms_win) / theo,
                     "l2": "flushed (256 MB write) between iterations" if small else "inputs > L2"})
        del q, k, v, out
        torch.cuda.empty_cache()
    return rows


TARGET_WORKLOADS = {"flux4096": "flux-4096px-256x256-w32", "wan720p": "wan-720p-21x45x80-w7x15x16"}


def targets_of(per_wl):
    """Compact summary of the two workloads the stated targets (>= 0.55 of peak,
    speedup >= 0.9 of N/n_w) apply to, from the per-workload table."""
    out = {}
    for key, name in TARGET_WORKLOADS.items():
        rows = [r for r in per_wl if r["workload"] == name]
        if not rows:
            continue
        r = rows[0]
        out[key] = {"ms_window": [round(x["ms"], 4) for x in r["window"]],
                    "tflops": round(r["flops_window"] / r["ms_window_mean"] / 1e9, 1),
                    "frac_of_peak": round(statistics.mean(x["frac_of_peak"] for x in r["window"]), 4),
                    "ms_full": round(r["ms_full"], 3), "full_frac_of_peak": round(r["full_frac_of_peak"], 4),
                    "speedup_vs_full": round(r["speedup_vs_full"], 2),
                    "speedup_frac_of_theoretical": round(r["speedup_frac_of_theoretical"], 4)}
    return out


def text_memory_case(stream, device, peak_tflops, n_text=512, pool=(1, 4, 4)):
    """FLUX-like joint attention on the 4096^2 image grid: every visual query
    attends to its window, n_text text tokens and the pooled memory of K and V
    (one extra segment [text; pooled]).  Times the pooling and the forward."""
    import torch
    import shifted_window_attention_swattn_b200 as sw
    from shifted_window_attention_swattn_b200.inputs import BY_NAME, make_custom, make_qkv
    wl = BY_NAME[TARGET_WORKLOADS["flux4096"]]
    q, k, v = make_qkv(wl, device=device)
    kt, vt, _ = make_custom(wl.B, wl.heads, wl.d, 1, 1, n_text, seed=4343, device=device)
    G = sw.kv_pool_tokens(wl.grid, pool)
    kx = torch.empty((wl.B, n_text + G, wl.heads, wl.d), dtype=torch.bfloat16, device=device)
    vx = torch.empty_like(kx)
    kx[:, :n_text] = kt
    vx[:, :n_text] = vt
    out = torch.empty_like(q)
    shift = wl.shifts[1]

    def pool_step():
        kbar, vbar = sw.kv_pool(k, v, wl.grid, pool, stream=stream)
        kx[:, n_text:] = kbar
        vx[:, n_text:] = vbar

    def fwd():
        sw.swattn_fwd_mem(q, k, v, kx, vx, wl.grid, wl.win, shift, wl.scale, out=out, stream=stream)
    with torch.cuda.stream(stream):
        pool_step()
    time_launches(fwd, 3, stream)
    ms_fwd = statistics.median(time_launches(fwd, 20, stream))
    E = n_text + G
    f_fwd = sw.flops(wl.B, wl.heads, wl.grid, wl.d, wl.win) + 4.0 * wl.B * wl.heads * wl.d * wl.N * E
    return {"workload": wl.name, "shift_thw": list(shift), "text_tokens": n_text, "pool_thw": list(pool),
            "pooled_tokens": G, "extra_tokens": E, "ms_fwd": ms_fwd, "flops_fwd": f_fwd,
            "tflops_fwd": f_fwd / ms_fwd / 1e9, "frac_of_peak": f_fwd / ms_fwd / 1e9 / peak_tflops}


def run_native(args):
    import torch
    import torch.distributed as dist
    import shifted_window_attention_swattn_b200 as sw
    from shifted_window_attention_swattn_b200.inputs import BY_NAME, make_qkv

    rank, world, local = dist_env()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    def barrier():
        if world > 1:
            dist.barrier()

    peaks, peak_src = load_peaks()
    peak_tflops = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    wl = BY_NAME[args.workload]
    if args.heads:
        # a smaller case of the same workload (profiling captures): fewer heads,
        # the same grid, windows and shifts
        wl = dataclasses.replace(wl, heads=args.heads)
    if args.full_attention:
        # the same kernel run as full attention (window = whole grid, no shift)
        wl = dataclasses.replace(wl, win=wl.grid, shifts=((0, 0, 0),))
    stream = torch.cuda.current_stream(device)
    q, k, v = make_qkv(wl, device=device, seed=wl.seed + 1000 * rank)
    out = torch.empty_like(q)
    f_layer = sw.flops(wl.B, wl.heads, wl.grid, wl.d, wl.win)
    f_step = f_layer * len(wl.shifts)

    def step():
        for shift in wl.shifts:
            sw.swattn_fwd(q, k, v, wl.grid, wl.win, shift, wl.scale, out=out, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if sw.last_device_error() != sw.BASA_OK:
        raise RuntimeError("device-side wait timed out during warm-up")

    # ---------------- timed region: exactly K steps
    with ClockSampler(local) as clocks:
        barrier()
        torch.cuda.synchronize()
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_total = ev0.elapsed_time(ev1)
    if sw.last_device_error() != sw.BASA_OK:
        raise RuntimeError("device-side wait timed out in the timed region")
    launches = args.steps * len(wl.shifts)
    t_max = max_over_ranks(ms_total, world, device)
    ms_per_step = t_max / args.steps
    value = whole_job_tflops(f_step * args.steps, world, t_max)
    ms_launch = ms_total / launches
    achieved = f_layer / (ms_launch / 1e3) / 1e12

    # ---------------- end to end from pinned host buffers, pipelined across steps
    # Every step copies its own Q, K, V from pinned host memory, runs the forward
    # for each shift and copies each output back.  Three streams (H2D copies,
    # compute, D2H copies) and two device buffer sets let step k+1's inputs come
    # in and step k-1's outputs go out while step k computes; events order each
    # buffer's reuse.  The timed region runs from before the first H2D copy to
    # after the last D2H copy.
    e2e = None
    if not args.no_e2e:
        q_h = q.cpu().pin_memory()
        k_h = k.cpu().pin_memory()
        v_h = v.cpu().pin_memory()
        outs_h = [torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True) for _ in wl.shifts]
        ins_d = [tuple(torch.empty_like(q) for _ in range(3)) for _ in range(2)]
        outs_d = [[torch.empty_like(q) for _ in wl.shifts] for _ in range(2)]
        s_in = torch.cuda.Stream(device=device)
        s_out = torch.cuda.Stream(device=device)
        ev = lambda: torch.cuda.Event()

        def e2e_run(n):
            computed = [None, None]   # per buffer set: the compute of its last step is done
            copied = [None, None]     # per buffer set: the D2H copies of its last step are done
            for it in range(n):
                b_ = it % 2
                qd, kd, vd = ins_d[b_]
                with torch.cuda.stream(s_in):
                    if computed[b_] is not None:
                        s_in.wait_event(computed[b_])
                    qd.copy_(q_h, non_blocking=True)
                    kd.copy_(k_h, non_blocking=True)
                    vd.copy_(v_h, non_blocking=True)
                    loaded = ev()
                    loaded.record(s_in)
                with torch.cuda.stream(stream):
                    stream.wait_event(loaded)
                    if copied[b_] is not None:
                        stream.wait_event(copied[b_])
                    for shift, od in zip(wl.shifts, outs_d[b_]):
                        sw.swattn_fwd(qd, kd, vd, wl.grid, wl.win, shift, wl.scale, out=od, stream=stream)
                    computed[b_] = ev()
                    computed[b_].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(computed[b_])
                    for oh, od in zip(outs_h, outs_d[b_]):
                        oh.copy_(od, non_blocking=True)
                    copied[b_] = ev()
                    copied[b_].record(s_out)
            done = ev()
            done.record(s_out)
            return done

        e2e_steps = max(3, min(args.steps, 10))
        e2e_run(2)
        torch.cuda.synchronize()
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        s_in.wait_stream(stream)
        done = e2e_run(e2e_steps)
        stream.wait_event(done)
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(a.elapsed_time(b), world, device)
        e2e = {"value": whole_job_tflops(f_step * e2e_steps, world, e2e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": 3 * q.numel() * 2,
               "d2h_bytes_per_step": len(wl.shifts) * q.numel() * 2,
               "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
               "path": "pinned host Q/K/V -> H2D (copy stream) -> basa_swattn_fwd per shift (compute "
                       "stream) -> D2H of each output (copy stream); two device buffer sets, so one "
                       "step's copies overlap the neighbouring steps' compute and copies"}
        del q_h, k_h, v_h, outs_h, ins_d, outs_d

    extras = {}
    cpu_base = None
    if rank == 0 and world == 1:
        # per-layer timing of each shift, and the full-attention comparison
        flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
        per_wl = sweep_workloads(stream, flush, peak_tflops) if not args.no_sweep else []
        extras["per_workload"] = per_wl
        if per_wl:
            extras["targets"] = targets_of(per_wl)
        head = [r for r in per_wl if r["workload"] == wl.name]
        if head:
            extras["speedup_vs_full"] = head[0]["speedup_vs_full"]
            extras["theoretical_speedup"] = head[0]["theoretical_speedup"]
            extras["speedup_frac_of_theoretical"] = head[0]["speedup_frac_of_theoretical"]
            extras["full_attention_ms"] = head[0]["ms_full"]
        del flush
        # An L-layer stack under the interleaved shift schedule (one forward per
        # layer, layer l shifted by the schedule's Delta_l).
        if args.schedule_layers > 0:
            shifts = sw.shift_schedule(args.schedule_layers, wl.win)

            def stack():
                for shift in shifts:
                    sw.swattn_fwd(q, k, v, wl.grid, wl.win, shift, wl.scale, out=out, stream=stream)
            time_launches(stack, 2, stream)
            ms_stack = statistics.median(time_launches(stack, 10, stream))
            extras["schedule"] = {
                "layers": len(shifts), "shifts_thw": [list(x) for x in shifts],
                "ms_per_stack": ms_stack, "ms_per_layer": ms_stack / len(shifts),
                "tflops": f_layer * len(shifts) / ms_stack / 1e9,
                "step_offset": [0, 0, 0]}
        # Pooled global memory (§3.2): pool K/V into G tokens per (b, head), then
        # the windowed forward with those G tokens appended to every window.
        if args.memory_pool:
            pool = tuple(int(x) for x in args.memory_pool.split(","))
            G = sw.kv_pool_tokens(wl.grid, pool)
            kbar, vbar = sw.kv_pool(k, v, wl.grid, pool, stream=stream)

            def pool_only():
                sw.kv_pool(k, v, wl.grid, pool, stream=stream)

            def fwd_mem():
                sw.swattn_fwd_mem(q, k, v, kbar, vbar, wl.grid, wl.win, wl.shifts[1], wl.scale,
                                  out=out, stream=stream)
            time_launches(fwd_mem, 2, stream)
            ms_mem = statistics.median(time_launches(fwd_mem, 10, stream))
            time_launches(pool_only, 2, stream)
            ms_pool = statistics.median(time_launches(pool_only, 10, stream))
            f_mem = f_layer + 4.0 * wl.B * wl.heads * wl.d * wl.N * G
            extras["memory"] = {
                "pool_thw": list(pool), "pooled_tokens": G, "shift_thw": list(wl.shifts[1]),
                "ms_pool": ms_pool, "ms_fwd": ms_mem, "flops_fwd": f_mem,
                "tflops_fwd": f_mem / ms_mem / 1e9,
                "pool_gbs": 2 * (wl.B * wl.N + wl.B * G) * wl.heads * wl.d * 2 / ms_pool / 1e6}
            del kbar, vbar
        # True-window routing (§3.3): window descriptors and top-1 routes, then
        # the forward over S_i = W_i u R_i u G (with the pooled memory above when
        # enabled), on the second shift of the workload.
        if args.route:
            import numpy as np
            shift = wl.shifts[1]
            nw = sw.n_windows(wl.grid, wl.win)
            ws = torch.empty(sw.route_workspace_bytes(wl.B, wl.heads, wl.grid, wl.d, wl.win), dtype=torch.uint8,
                             device=device)
            routed = torch.empty((wl.B, wl.heads, nw), dtype=torch.int32, device=device)

            def route_only():
                sw.route(q, k, wl.grid, wl.win, shift, 1, out=routed, workspace=ws, stream=stream)
            time_launches(route_only, 2, stream)
            ms_route = statistics.median(time_launches(route_only, 10, stream))
            pool = tuple(int(x) for x in args.memory_pool.split(",")) if args.memory_pool else None
            G = sw.kv_pool_tokens(wl.grid, pool) if pool else 0
            kbar, vbar = sw.kv_pool(k, v, wl.grid, pool, stream=stream) if pool else (None, None)

            def fwd_route():
                sw.swattn_fwd_route(q, k, v, routed, wl.grid, wl.win, shift, kbar, vbar, wl.scale, out=out,
                                    stream=stream)
            time_launches(fwd_route, 2, stream)
            ms_fwd_rt = statistics.median(time_launches(fwd_route, 10, stream))
            torch.cuda.synchronize()
            # FLOPs from the routes taken: 4 d per (query, key) pair, keys = own
            # window + routed window + G pooled tokens
            counts = (sw.index_map_host(wl.grid, wl.win, shift) >= 0).sum(axis=1).astype(np.float64)
            r = routed.cpu().numpy().reshape(-1, nw)
            n_rt = np.where(r >= 0, counts[np.clip(r, 0, None)], 0.0)
            f_rt = 4.0 * wl.d * float(np.sum(counts[None, :] * (counts[None, :] + n_rt + G)))
            extras["route"] = {
                "radius": 1, "top_k": 1, "shift_thw": list(shift), "windows": nw,
                "routed_fraction": float(np.mean(r >= 0)),
                "ms_route": ms_route,
                "route_gbs": 2 * wl.B * wl.N * wl.heads * wl.d * 2 / ms_route / 1e6,
                "pool_thw": list(pool) if pool else None, "pooled_tokens": G,
                "ms_fwd": ms_fwd_rt, "flops_fwd": f_rt, "tflops_fwd": f_rt / ms_fwd_rt / 1e9,
                "source": "own window + routed window" + (" + pooled memory" if pool else "")}
            del ws, routed, kbar, vbar
        if args.text_memory:
            extras["text_memory"] = text_memory_case(stream, device, peak_tflops)
            torch.cuda.empty_cache()
        # CPU baseline: the oracle on a bounded sample of the same workload
        if not args.no_cpu_baseline:
            qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
            threads = host_threads()
            t_probe, _, _ = oracle_rows_sample(wl, qc, kc, vc, threads * 2 * 4, threads, seed=1)
            rows_per_s = threads * 2 * 4 / max(t_probe, 1e-6)
            n_rows = int(max(threads * 2, min(rows_per_s * 12.0, 400000)))
            t_cpu, f_cpu, rows = oracle_rows_sample(wl, qc, kc, vc, n_rows, threads, seed=2)
            cpu_base = {"value": f_cpu / t_cpu / 1e12, "unit": "TFLOP/s", "cores": threads,
                        "kind": "oracle",
                        "sample": (f"{rows} random query rows of {wl.name} (both shifts), oracle "
                                   f"per-row path in fp64, {t_cpu:.1f} s on {threads} host "
                                   f"threads, CPU {cpu_model()}")}

    traffic_rec = load_traffic()
    # the recorded traffic is that of the default headline configuration
    custom = bool(args.heads) or args.full_attention or args.workload != HEADLINE
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": wl_config(wl, {"parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                                 **({"mode": "full attention"} if args.full_attention else {})}),
        "frac_of_peak": achieved / peak_tflops,
        "peak_source": f"{peak_src} bf16 dense burst ({peak_tflops:.1f} TFLOP/s)",
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_tflops,
                     "unit": "TFLOP/s", "frac": achieved / peak_tflops,
                     "traffic": traffic_rec["dram_bytes_per_launch"] if traffic_rec and not custom else None,
                     "kernel": KERNEL_NAME if wl.d == 128 else "swattn_fwd_kernel",
                     "flops_per_launch": f_layer,
                     "ms_per_launch": ms_launch,
                     "peak_kind": f"{peak_src} burst"},
        "cpu_baseline": cpu_base,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    # the compact target summary goes right after the configuration, the long
    # per-workload table last
    if "targets" in extras:
        line = dict(list(line.items())[:13] + [("targets", extras.pop("targets"))] + list(line.items())[13:])
    per_wl = extras.pop("per_workload", None)
    line.update(extras)
    if per_wl is not None:
        line["per_workload"] = per_wl
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--no-sweep", action="store_true", help="skip the per-workload table")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end timing")
    ap.add_argument("--memory-pool", default="1,4,4",
                    help="also time the pooled global memory: pooling factors t,h,w ('' to skip)")
    ap.add_argument("--route", action=argparse.BooleanOptionalAction, default=True,
                    help="time true-window routing and the routed forward (the `route` key)")
    ap.add_argument("--text-memory", action=argparse.BooleanOptionalAction, default=True,
                    help="time the FLUX-like joint attention: window + 512 text tokens + pooled memory "
                         "(the `text_memory` key)")
    ap.add_argument("--schedule-layers", type=int, default=8,
                    help="also time an L-layer stack under the interleaved shift schedule (0: off)")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the workload's head count (a smaller case of it, for profiling captures)")
    ap.add_argument("--full-attention", action="store_true",
                    help="run the step in full-attention mode (window = grid, shift 0), for profiling captures")
    ap.add_argument("--workload", default=HEADLINE,
                    help="workload name from shifted_window_attention_swattn_b200.inputs "
                         "(profiling runs of a smaller case; the default is the headline)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
