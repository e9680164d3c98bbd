#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200: one step = fa_fwd + fa_bwd.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Workload (default): causal, B=2, H=16, N=8192, d=128, bf16 -- the forward +
recompute-backward configuration.  Inputs are seeded synthetic N(0,1) bf16
(``exact_io_aware_93_b200.inputs``), resident in HBM before the timed region.
Q, K, V, dO, O together exceed the 126 MB L2, so L2 is not flushed between steps.

Prints ONE JSON line (rank 0).  ``value`` is whole-job TFLOPS under the FLOP
convention forward = 4*B*H*N^2*d (halved when causal), backward = 2.5x forward,
summed over all ranks.  With N > 1 (torchrun) every rank runs the same workload
on its own GPU (independent replicas, weak scaling, no data-path collective);
the time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle (the slow, plain definition the
parity tests use) on the host cores, each step one full head of the same
workload (forward and backward), and prints the same JSON line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_io_aware_93_b200.accounting import (bwd_flops_window, decode_bytes, decode_flops, fwd_bytes,  # noqa: E402
                                                fwd_flops_window)
from exact_io_aware_93_b200.inputs import (DECODE_WORKLOADS, EXTRA_WORKLOADS, WORKLOADS,  # noqa: E402
                                           make_decode_workload_inputs, make_inputs, make_workload_inputs)
from exact_io_aware_93_b200.replicas import max_over_ranks, whole_job_tflops, world as _world  # noqa: E402

METRIC = "attention fwd/bwd TFLOPS and % of B200 dense-bf16 peak, causal N=2K–128K"
NOMINAL_BF16_TFLOPS = 2250.0   # datasheet dense bf16 per GPU (the 2:4-sparse figure halved)
DECODE_METRIC = "attention decode: key/value cache bytes streamed per second (GB/s) and % of B200 HBM bandwidth"
DEFAULT_WORKLOAD = "causal_fwdbwd_b2_h16_n8192_d128"
FWD_ALONE_PAUSE_S = 1.0        # idle time before the forward-alone burst
L2_BYTES = 126 * 1024 * 1024


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), \
            float(p["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, 1400.0, 6650.0, "fallback"


def kernel_source_digest() -> str:
    """Digest of the CUDA sources; ncu traffic figures are valid only for the digest they name."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_93_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, or None if absent or stale."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
    except (OSError, ValueError):
        return None
    rec = table.get(kernel, {}).get(workload)
    if not rec or rec.get("source_digest") != kernel_source_digest():
        return None
    return rec.get("dram_bytes_per_launch")


def _dist_env():
    return _world()


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples, kept only when taken inside the timed region."""

    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"fa_bench_clocks_{os.getpid()}.csv")
        self.window = None

    def start(self):
        """Start sampling; returns once the first sample has arrived (or after 3 s)."""
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.QUERY}", "--format=csv,noheader",
                 "-lms", "20"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        t0 = time.time()
        while time.time() - t0 < 3.0 and os.path.getsize(self.path) == 0:
            time.sleep(0.02)

    def mark(self, t_begin: float, t_end: float):
        self.window = (t_begin, t_end)

    def stop(self):
        """End sampling and return the statistics of the window given to mark()."""
        self.close()
        return self.stats(self.window)

    def close(self):
        """End sampling and read every sample; stats() then summarises any window."""
        self.samples = []
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        with open(self.path) as f:
            self.samples = parse_clock_samples(f)
        os.unlink(self.path)

    def stats(self, window):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0, "power_cap_samples": 0,
                    "reasons": ["nvidia-smi unavailable"]}
        return clock_stats(self.samples, window)


CLOCK_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


def parse_clock_samples(lines):
    """Rows of the nvidia-smi query above as dicts (timestamp in seconds since the epoch)."""
    import datetime
    out = []
    for line in lines:
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 10:
            continue
        try:
            ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            clk, cmax = float(parts[2].split()[0]), float(parts[3].split()[0])
            pw = float(parts[4].split()[0])
        except ValueError:
            continue
        out.append({"ts": ts, "sm": clk, "sm_max": cmax, "power": pw,
                    "reasons": [n for n, v in zip(CLOCK_REASONS, parts[6:10]) if v.lower() == "active"]})
    return out


def clock_stats(samples, window, slack_s: float = 0.05):
    """Median SM clock, max clock, peak power and the throttle reasons of the samples taken
    inside `window` (t_begin, t_end), with the number of samples that saw the power cap."""
    sel = [x for x in samples if window is None or window[0] - slack_s <= x["ts"] <= window[1] + slack_s]
    reasons = sorted({r for x in sel for r in x["reasons"]})
    return {"sm_mhz": statistics.median(x["sm"] for x in sel) if sel else None,
            "sm_max_mhz": max(x["sm_max"] for x in sel) if sel else None,
            "power_w_max": max(x["power"] for x in sel) if sel else None,
            "samples": len(sel),
            "power_cap_samples": sum("sw_power_cap" in x["reasons"] for x in sel),
            "reasons": reasons}


def choose_peak(clk, burst: float, sustained: float):
    """The tensor peak a timed region is compared with, chosen from that region's own clock
    samples: the sustained (power-capped) cuBLAS figure when more than half of the in-region
    samples show sw_power_cap, else the burst figure (the larger denominator: a region that
    ran mostly uncapped is not excused by a capped sample or two).  Returns
    (peak, kind, rule)."""
    n, capped = clk.get("samples", 0) or 0, clk.get("power_cap_samples", 0) or 0
    rule = f"sw_power_cap active in {capped} of {n} in-region clock samples"
    if n > 0 and 2 * capped > n:
        return sustained, "sustained", rule + " (a majority)"
    return burst, "burst", rule + (" (not a majority)" if capped else "")


def pipelined_e2e(sets, host_in, in_names, out_names, compute, nsteps):
    """Mean milliseconds per step of `nsteps` end-to-end steps.  Every step copies its inputs
    in from pinned host memory, runs `compute(buffer_set)` and copies its results out to
    pinned host memory.  Steps are pipelined the way a training or serving loop runs them:
    while step i computes, step i+1's inputs come in and step i-1's results go out (two device
    buffer sets, three streams ordered by events; a buffer set is refilled only after the step
    two back has finished reading it and its results have left)."""
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    host_out = {n: torch.empty(sets[0][n].shape, dtype=sets[0][n].dtype).pin_memory() for n in out_names}
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(s_in)
    comp_done, out_done = [None, None], [None, None]
    for i in range(nsteps):
        b = sets[i % 2]
        with torch.cuda.stream(s_in):
            if comp_done[i % 2] is not None:
                s_in.wait_event(comp_done[i % 2])
            for n in in_names:
                b[n].copy_(host_in[n], non_blocking=True)
            in_done = torch.cuda.Event()
            in_done.record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done)
            if out_done[i % 2] is not None:
                s_comp.wait_event(out_done[i % 2])
            compute(b)
            comp_done[i % 2] = torch.cuda.Event()
            comp_done[i % 2].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[i % 2])
            for n in out_names:
                host_out[n].copy_(b[n], non_blocking=True)
            out_done[i % 2] = torch.cuda.Event()
            out_done[i % 2].record(s_out)
    f1.record(s_out)
    torch.cuda.synchronize()
    return f0.elapsed_time(f1) / nsteps


def _win(w):
    return None if w.window < 0 else w.window


def fwd_flops(B, H, N, d, causal, window=-1):
    return fwd_flops_window(B, H, N, d, causal, window)


def bwd_flops(B, H, N, d, causal, window=-1):
    return bwd_flops_window(B, H, N, d, causal, window)


def _step_fn(api, t, w, with_bwd, events=None):
    """One pass of the hot path: fa_fwd then (if available) fa_bwd, on the current stream."""
    def step():
        if events is not None:
            events["fwd"].append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
            events["fwd"][-1][0].record()
        if w.dtype == "e4m3":
            api.fwd_e4m3(t["q"], t["k"], t["v"], t["q_descale"], t["k_descale"], t["v_descale"],
                         causal=w.causal, out=t["o"], lse=t["lse"], window=_win(w))
        else:
            api.fwd(t["q"], t["k"], t["v"], causal=w.causal, out=t["o"], lse=t["lse"], window=_win(w))
        if events is not None:
            events["fwd"][-1][1].record()
        if with_bwd:
            if events is not None:
                events["bwd"].append((torch.cuda.Event(enable_timing=True),
                                      torch.cuda.Event(enable_timing=True)))
                events["bwd"][-1][0].record()
            api.bwd(t["q"], t["k"], t["v"], t["o"], t["do"], t["lse"], causal=w.causal,
                    dq=t["dq"], dk=t["dk"], dv=t["dv"], workspace=t["ws"], window=_win(w))
            if events is not None:
                events["bwd"][-1][1].record()
    return step


def cpu_sample(w, heads: int, threads: int, rows: int | None = None, backward: bool = True):
    """Time the fp64 oracle on `heads` heads of workload w.

    rows=None: every query row of each head; otherwise the forward of the last `rows` query
    rows (the rows that see the most keys).  backward=True adds the full-head backward.
    Returns (FLOPs under the benchmark's convention, seconds).
    """
    import oracle
    oracle.oracle_threads(threads)
    inp = make_inputs(1, heads, w.N, w.d, w.seed, with_do=backward)
    sel = None if rows is None else list(range(w.N - rows, w.N))
    t0 = time.perf_counter()
    flops = 0.0
    for h in range(heads):
        q, k, v = (inp[n][0, :, h].double().numpy() for n in ("q", "k", "v"))
        oracle.fwd_rows(q, k, v, w.scale, w.causal, sel, window=w.window)
        if sel is None:
            flops += fwd_flops(1, 1, w.N, w.d, w.causal, w.window)
        else:
            flops += sum(4.0 * ((min(i, w.window) + 1 if w.window >= 0 else i + 1) if w.causal else w.N) * w.d
                         for i in sel)
        if backward:
            do = inp["do"][0, :, h].double().numpy()
            oracle.bwd_rows(q, k, v, do, w.scale, w.causal, window=w.window)
            flops += bwd_flops(1, 1, w.N, w.d, w.causal, w.window)
    dt = time.perf_counter() - t0
    return flops, dt


def with_bwd_available() -> bool:
    try:
        from exact_io_aware_93_b200 import api
        return hasattr(api.lib(), "fa_bwd") and hasattr(api, "bwd")
    except (FileNotFoundError, OSError):
        return False


REFERENCE_BUDGET_S = 150.0


def run_reference(args, w):
    """The fp64 oracle on the host cores, each step a sample of the same workload sized so the
    whole run (warm-up + timed steps) stays within about REFERENCE_BUDGET_S seconds."""
    world, rank, _ = _dist_env()
    if rank != 0:
        return 0
    threads = len(os.sched_getaffinity(0))
    per_step = REFERENCE_BUDGET_S / (args.warmup + args.steps)
    # calibrate the oracle's rate on a small forward sample
    cf, ct = cpu_sample(w, 1, threads, rows=256, backward=False)
    rate = cf / ct
    full = fwd_flops(1, 1, w.N, w.d, w.causal) + (bwd_flops(1, 1, w.N, w.d, w.causal) if w.backward else 0.0)
    if full / rate <= per_step:
        kw = {"rows": None, "backward": w.backward}
        sample = f"1 full head (b=0, h=0) of {w.name}: forward" + (" and backward" if w.backward else "") \
                 + " of every row, fp64"
    else:
        rows = w.N
        while rows > 64 and sum(4.0 * ((i + 1) if w.causal else w.N) * w.d
                                for i in range(w.N - rows, w.N)) / rate > per_step:
            rows //= 2
        kw = {"rows": None if rows == w.N else rows, "backward": False}
        sample = (f"forward of the last {rows} query rows of head (b=0, h=0) of {w.name}, fp64 "
                  f"(backward left out so {args.warmup + args.steps} steps fit ~{REFERENCE_BUDGET_S:.0f} s)")
    times = []
    flops_step = 0.0
    for i in range(args.warmup + args.steps):
        flops_step, dt = cpu_sample(w, 1, threads, **kw)
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = flops_step * len(times) / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _device_inputs(api, w, dev, with_bwd):
    """Seeded inputs of workload w on the device plus its output buffers and workspace."""
    is8 = w.dtype == "e4m3"
    if is8:
        inp = make_workload_inputs(w)
        names = ("q", "k", "v")
    else:
        inp = make_inputs(w.B, w.H, w.N, w.d, w.seed, with_do=True, peaked=w.peaked, H_kv=w.H_kv,
                          dtype=w.torch_dtype)
        names = ("q", "k", "v", "do")
    t = {n: inp[n].to(dev) for n in names}
    if is8:
        t.update({n: inp[n] for n in ("q_descale", "k_descale", "v_descale")})
    t["o"] = torch.empty(t["q"].shape, dtype=torch.bfloat16 if is8 else t["q"].dtype, device=dev)
    t["lse"] = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    if with_bwd:
        t["dq"], t["dk"], t["dv"] = torch.empty_like(t["q"]), torch.empty_like(t["k"]), torch.empty_like(t["v"])
        t["ws"] = torch.empty(api.bwd_workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
    return inp, t, names


def _timed_steps(api, t, w, with_bwd, nsteps, barrier=None):
    """Time `nsteps` back-to-back steps with CUDA events on the launch stream.  Returns the
    wall-clock window (for the clock samples), the mean step time and the mean forward and
    backward times from per-step events."""
    events = {"fwd": [], "bwd": []}
    tstep = _step_fn(api, t, w, with_bwd, events)
    if barrier is not None:
        barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_begin = time.time()
    e0.record()
    for _ in range(nsteps):
        tstep()
    e1.record()
    torch.cuda.synchronize()
    t_end = time.time()
    ms = e0.elapsed_time(e1) / nsteps
    fwd_ms = statistics.mean(a.elapsed_time(b) for a, b in events["fwd"])
    bwd_ms = statistics.mean(a.elapsed_time(b) for a, b in events["bwd"]) if events["bwd"] else None
    ends = events["bwd"] if events["bwd"] else events["fwd"]
    per_step = sorted(f[0].elapsed_time(e[1]) for f, e in zip(events["fwd"], ends))
    return {"window": (t_begin, t_end), "ms": ms, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "per_step": per_step}


# The metric's sequence-length range: a fwd + bwd step of each causal configuration, each
# timed for about PER_CONFIG_SECONDS with its own clock record.
PER_CONFIG = ("causal_b4_h16_n2048_d128", "causal_fwdbwd_b2_h16_n8192_d128", "causal_b1_h32_n32768_d128",
              "causal_peaked_b1_h8_n131072_d128")
PER_CONFIG_SECONDS = 1.0


def per_config_records(api, dev, clocks, burst, sustained, warmup):
    """One record per PER_CONFIG workload: fwd_ms, bwd_ms, the step's TFLOP/s and the
    fraction of the peak its own in-region clock samples select (choose_peak)."""
    out = {}
    for name in PER_CONFIG:
        w = WORKLOADS[name]
        inp, t, _ = _device_inputs(api, w, dev, True)
        del inp
        step = _step_fn(api, t, w, True)
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record()
        for _ in range(warmup):
            step()
        g1.record()
        torch.cuda.synchronize()
        est_ms = g0.elapsed_time(g1) / warmup
        nsteps = max(5, min(500, int(PER_CONFIG_SECONDS * 1e3 / max(est_ms, 1e-3))))
        r = _timed_steps(api, t, w, True, nsteps)
        out[name] = r
        out[name]["steps"] = nsteps
        out[name]["status"] = api.get_status()
        del t
        torch.cuda.empty_cache()
    return out


def _per_config_json(recs, clocks, burst, sustained):
    js = {}
    for name, r in recs.items():
        w = WORKLOADS[name]
        ff = fwd_flops(w.B, w.H, w.N, w.d, w.causal, w.window)
        fb = bwd_flops(w.B, w.H, w.N, w.d, w.causal, w.window)
        clk = clocks.stats(r["window"])
        peak, kind, rule = choose_peak(clk, burst, sustained)
        step_tf = (ff + fb) / (r["ms"] * 1e-3) / 1e12
        fwd_tf = ff / (r["fwd_ms"] * 1e-3) / 1e12
        bwd_tf = fb / (r["bwd_ms"] * 1e-3) / 1e12
        js[name] = {"B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "peaked": w.peaked,
                    "steps": r["steps"], "ms_per_step": r["ms"], "fwd_ms": r["fwd_ms"], "bwd_ms": r["bwd_ms"],
                    "step_tflops": step_tf, "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
                    "peak": peak, "peak_kind": kind, "peak_rule": rule,
                    "step_frac": step_tf / peak, "fwd_frac": fwd_tf / peak, "bwd_frac": bwd_tf / peak,
                    "clocks": clk, "device_status": r["status"]}
    return js


def run_ours(args, w):
    world, rank, local = _dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from exact_io_aware_93_b200 import api
    dev = torch.device("cuda", torch.cuda.current_device())
    is8 = w.dtype == "e4m3"             # the e4m3 path is forward only
    with_bwd = with_bwd_available() and not is8
    inp, t, names = _device_inputs(api, w, dev, with_bwd)
    in_bytes = sum(t[n].numel() * t[n].element_size() for n in names)

    step = _step_fn(api, t, w, with_bwd)
    clocks = ClockSampler(dev.index)
    clocks.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if api.get_status() != 0:
        raise RuntimeError("device status word set during warm-up")

    # ---------------- device-timed region
    barrier = None
    if world > 1:
        import torch.distributed as dist
        barrier = dist.barrier
    r = _timed_steps(api, t, w, with_bwd, args.steps, barrier)
    if world > 1:
        dist.barrier()
    ms, fwd_ms, bwd_ms, per_step = r["ms"], r["fwd_ms"], r["bwd_ms"], r["per_step"]
    pct = lambda q: per_step[min(len(per_step) - 1, int(q * len(per_step)))]
    step_dist = {"p10_ms": pct(0.10), "median_ms": pct(0.50), "p90_ms": pct(0.90)}
    status = api.get_status()

    # ---------------- the forward pass on its own (same inputs, back to back): the rate the
    # forward target refers to, next to its rate inside the fwd + bwd step above
    fwd_only = None
    if with_bwd:
        def fwd_step():
            _step_fn(api, t, w, False)()
        # Timed as a burst, the way the burst peak it is compared with was measured: after a
        # short idle pause rather than straight after the step loop above.
        time.sleep(FWD_ALONE_PAUSE_S)
        for _ in range(3):
            fwd_step()
        torch.cuda.synchronize()
        fonly_steps = max(3, min(args.steps, 100))
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record()
        for _ in range(fonly_steps):
            fwd_step()
        g1.record()
        torch.cuda.synchronize()
        fwd_only = {"ms": g0.elapsed_time(g1) / fonly_steps, "steps": fonly_steps}

    # ---------------- end-to-end through the public API: pinned host in, results back
    host = {n: inp[n].pin_memory() for n in names}
    out_names = ["o", "lse"] + (["dq", "dk", "dv"] if with_bwd else [])
    d2h_bytes = sum(t[n].numel() * t[n].element_size() for n in out_names)
    e2e_steps = max(2, min(args.steps, 20))
    # a second device buffer set (the workspace is shared: the compute stream runs one step
    # at a time)
    t2 = {n: (torch.empty_like(x) if isinstance(x, torch.Tensor) and n != "ws" else x) for n, x in t.items()}
    sets = [t, t2]

    def compute(b):
        _step_fn(api, b, w, with_bwd)()

    pipelined_e2e(sets, host, names, out_names, compute, 2)   # warm-up
    if world > 1:
        dist.barrier()
    e2e_ms = pipelined_e2e(sets, host, names, out_names, compute, e2e_steps)

    if world > 1:
        ms, e2e_ms, fwd_ms, bwd_ms = max_over_ranks([ms, e2e_ms, fwd_ms, bwd_ms or 0.0], dev)
        bwd_ms = bwd_ms if with_bwd else None
        if fwd_only is not None:
            fwd_only["ms"] = max_over_ranks([fwd_only["ms"]], dev)[0]

    peak, peak_sus, hbm, peak_kind = _peaks()
    if is8:
        # e4m3 contraction: the measured bf16 peak times the nominal dense e4m3 / bf16 ratio (2)
        peak, peak_sus, peak_kind = 2 * peak, 2 * peak_sus, peak_kind + " bf16 x 2 (nominal e4m3/bf16 ratio);"

    # ---------------- the metric's range: N = 2K, 8K, 32K, 128K, each with its own clocks
    recs = None
    if world == 1 and not args.no_per_config and w.name == DEFAULT_WORKLOAD and with_bwd:
        del t2, sets
        torch.cuda.empty_cache()
        recs = per_config_records(api, dev, clocks, peak, peak_sus, 3)
    clocks.close()
    clk = clocks.stats(r["window"])

    ff = fwd_flops(w.B, w.H, w.N, w.d, w.causal, w.window)
    fb = bwd_flops(w.B, w.H, w.N, w.d, w.causal, w.window) if with_bwd else 0.0
    step_flops = ff + fb
    value = whole_job_tflops(world, step_flops, ms)
    e2e_value = whole_job_tflops(world, step_flops, e2e_ms)
    fwd_tf = ff / (fwd_ms * 1e-3) / 1e12
    bwd_tf = fb / (bwd_ms * 1e-3) / 1e12 if with_bwd else None
    # dominant kernel: the one with the larger share of the step
    if with_bwd and bwd_ms > fwd_ms:
        dom = {"kernel": "fa_bwd (pre + main + post)", "achieved": bwd_tf, "ms": bwd_ms, "key": "fa_bwd"}
    else:
        dom = {"kernel": "fa_fwd_kernel", "achieved": fwd_tf, "ms": fwd_ms, "key": "fa_fwd_kernel"}
    # The denominator follows the timed region's own clock samples: the sustained
    # (power-capped) cuBLAS figure if any of them shows sw_power_cap, else the burst figure.
    chosen, chosen_kind, rule = choose_peak(clk, peak, peak_sus)
    roofline = {"bound": "tensor", "achieved": dom["achieved"], "peak": chosen, "unit": "TFLOP/s",
                "frac": dom["achieved"] / chosen, "traffic": measured_traffic(dom["key"], w.name),
                "kernel": dom["kernel"],
                "peak_kind": f"{peak_kind} bf16 {chosen_kind} (cuBLAS bf16 8192^3"
                             + (", back to back at the power cap)" if chosen_kind == "sustained" else ", burst)")
                             + (" x 2 for e4m3" if is8 else ""),
                "peak_rule": rule, "burst_peak": peak, "sustained_peak": peak_sus,
                "frac_of_burst": dom["achieved"] / peak, "frac_of_sustained": dom["achieved"] / peak_sus,
                "fwd_alg_bytes": fwd_bytes(w.B, w.H, w.N, w.d)}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
                   "H_kv": w.H_kv or w.H, "window": w.window,
                   "parallelism": f"replicas x{world}",
                   "l2": f"not flushed: inputs {in_bytes / 1e6:.0f} MB > L2 {L2_BYTES / 1e6:.0f} MB",
                   "step": "fa_fwd + fa_bwd" if with_bwd else
                           ("fa_fwd_e4m3_scaled (the e4m3 path is forward only)" if is8 else
                            "fa_fwd only (backward not built)")},
        "fwd_tflops": fwd_tf, "fwd_ms": fwd_ms, "bwd_tflops": bwd_tf, "bwd_ms": bwd_ms,
        "fwd_alone": None if fwd_only is None else {
            "tflops": ff / (fwd_only["ms"] * 1e-3) / 1e12, "ms": fwd_only["ms"], "steps": fwd_only["steps"],
            "pct_of_peak": 100.0 * ff / (fwd_only["ms"] * 1e-3) / 1e12 / peak,
            "note": f"fa_fwd alone, back to back on the same inputs, a short burst after a {FWD_ALONE_PAUSE_S:g} s idle pause: against the burst peak; "
                    "fwd_tflops is its rate inside the step"},
        "pct_of_peak": 100.0 * value / world / peak,
        "pct_of_sustained_peak": 100.0 * value / world / peak_sus,
        "pct_of_nominal_peak": 100.0 * value / world / (NOMINAL_BF16_TFLOPS * (2 if is8 else 1)),
        "step_ms_distribution": step_dist,
        "roofline": roofline,
        "e2e": {"value": e2e_value, "unit": "TFLOPS", "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": d2h_bytes, "ms_per_step": e2e_ms, "steps": e2e_steps,
                "note": "every step copies its inputs in and all results out; steps pipelined on "
                        "three streams (copy-in, compute, copy-out)"},
        "gpu_launches": args.steps * (1 + (3 if with_bwd else 0)),
        "clocks": clk,
        "device_status": status,
    }
    if recs is not None:
        line["per_config"] = _per_config_json(recs, clocks, peak, peak_sus)
        line["per_config_note"] = (f"fa_fwd + fa_bwd steps of each causal configuration, each timed back to back "
                                   f"for about {PER_CONFIG_SECONDS:g} s after 3 warm-up steps, with the clock "
                                   "samples of its own timed window; *_frac use the peak those samples select "
                                   "(peak_rule)")
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = len(os.sched_getaffinity(0))
        heads = 4
        cflops, cdt = cpu_sample(w, heads, threads, backward=with_bwd)
        line["cpu_baseline"] = {
            "value": cflops / cdt / 1e12, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
            "extrapolated_full_step_s": step_flops / (cflops / cdt),
            "sample": f"{heads} full heads of {w.name} (forward" + (" + backward" if with_bwd else "")
                      + f", fp64{'; bf16-drawn inputs, the oracle costs the same for any input type' if is8 else ''}),"
                      f" {cdt:.1f} s"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def _decode_sample_heads(w, count):
    return [(b % w.B, (7 * b + 3) % w.H) for b in range(count)]


def decode_cpu_sample(w, inp, pairs, threads):
    """Time the fp64 oracle's decode on the given (b, h) pairs; returns (bytes, seconds) with
    bytes counted like decode_bytes for those heads (each head's key/value rows once)."""
    import oracle
    oracle.oracle_threads(threads)
    q, k, v = (inp[n].double().numpy() for n in ("q", "k", "v"))
    lens = inp["seqlens"].numpy()
    t0 = time.perf_counter()
    oracle.decode_rows(q, k, v, lens, w.scale, w.causal, w.window, heads=pairs)
    dt = time.perf_counter() - t0
    nbytes = sum(decode_bytes([lens[b]], 1, 1, 1, w.N_q, w.d, w.causal, w.window) for b, _ in pairs)
    return nbytes, dt


def run_decode(args, w):
    """Decoding workload: one step = one fa_decode call (split-KV kernel + merge kernel)."""
    world, rank, local = _dist_env()
    if args.impl == "reference":
        if rank != 0:
            return 0
        threads = len(os.sched_getaffinity(0))
        inp = make_decode_workload_inputs(w)
        per_step = REFERENCE_BUDGET_S / (args.warmup + args.steps)
        nb, dt = decode_cpu_sample(w, inp, _decode_sample_heads(w, 1), threads)
        heads = max(1, min(w.B * w.H, int(per_step / max(dt, 1e-6))))
        pairs = _decode_sample_heads(w, heads)
        times, nbytes = [], 0
        for i in range(args.warmup + args.steps):
            nbytes, dt = decode_cpu_sample(w, inp, pairs, threads)
            if i >= args.warmup:
                times.append(dt)
        value = nbytes * len(times) / sum(times) / 1e9
        line = {
            "impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "H_kv": w.H_kv, "N_q": w.N_q, "N_kv": w.N_kv,
                       "d": w.d, "causal": w.causal, "window": w.window},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": f"oracle decode of {len(pairs)} (sequence, head) pairs of {w.name} per step"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return 0
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from exact_io_aware_93_b200 import api
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = make_decode_workload_inputs(w)
    t = {n: inp[n].to(dev) for n in ("q", "k", "v", "seqlens")}
    t["o"] = torch.empty_like(t["q"])
    t["lse"] = torch.empty((w.B, w.H, w.N_q), dtype=torch.float32, device=dev)
    t["ws"] = torch.empty(api.decode_workspace_size(t["q"], t["k"], w.causal, _win(w)), dtype=torch.uint8,
                          device=dev)
    lens = inp["seqlens"].tolist()
    step_bytes = decode_bytes(lens, w.B, w.H, w.H_kv, w.N_q, w.d, w.causal, w.window)
    step_flops = decode_flops(lens, w.H, w.N_q, w.d, w.causal, w.window)
    cache_bytes = 2 * t["k"].numel() * t["k"].element_size()

    def step():
        api.decode(t["q"], t["k"], t["v"], t["seqlens"], causal=w.causal, out=t["o"], lse=t["lse"],
                   workspace=t["ws"], window=_win(w))

    clocks = ClockSampler(dev.index)
    clocks.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if api.get_status() != 0:
        raise RuntimeError("device status word set during warm-up")
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_begin = time.time()
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    t_end = time.time()
    if world > 1:
        dist.barrier()
    clocks.mark(t_begin, t_end)
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    status = api.get_status()

    # end to end through the public API: the new queries and lengths come from pinned host
    # memory and O, LSE go back every step; the cache stays resident on the device
    host_in = {n: inp[n].pin_memory() for n in ("q", "seqlens")}
    h2d = sum(x.numel() * x.element_size() for x in host_in.values())
    d2h = sum(t[n].numel() * t[n].element_size() for n in ("o", "lse"))
    t2 = dict(t)
    for n in ("q", "seqlens", "o", "lse"):
        t2[n] = torch.empty_like(t[n])

    def compute(b):
        api.decode(b["q"], b["k"], b["v"], b["seqlens"], causal=w.causal, out=b["o"], lse=b["lse"],
                   workspace=b["ws"], window=_win(w))

    e2e_steps = max(2, min(args.steps, 50))
    pipelined_e2e([t, t2], host_in, ("q", "seqlens"), ("o", "lse"), compute, 2)   # warm-up
    e2e_ms = pipelined_e2e([t, t2], host_in, ("q", "seqlens"), ("o", "lse"), compute, e2e_steps)
    if world > 1:
        ms, e2e_ms = max_over_ranks([ms, e2e_ms], dev)
    _, _, hbm, peak_kind = _peaks()
    gbs = step_bytes / (ms * 1e-3) / 1e9
    value = world * gbs
    line = {
        "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "H_kv": w.H_kv, "N_q": w.N_q, "N_kv": w.N_kv,
                   "d": w.d, "causal": w.causal, "window": w.window, "seqlens": lens,
                   "parallelism": f"replicas x{world}",
                   "l2": f"not flushed: key/value cache {cache_bytes / 1e6:.0f} MB > L2 {L2_BYTES / 1e6:.0f} MB",
                   "step": "fa_decode (split-KV kernel + merge kernel)"},
        "tokens_per_s": world * w.B * w.N_q / (ms * 1e-3),
        "tflops": world * step_flops / (ms * 1e-3) / 1e12,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "traffic": measured_traffic("fa_decode", w.name), "kernel": "fa_decode (kernel + merge)",
                     "peak_kind": f"{peak_kind} HBM copy bandwidth", "alg_bytes_per_launch": step_bytes},
        "e2e": {"value": world * step_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps},
        "gpu_launches": args.steps * 2,
        "clocks": clk,
        "device_status": status,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = len(os.sched_getaffinity(0))
        pairs = _decode_sample_heads(w, 16)
        nb, dt = decode_cpu_sample(w, inp, pairs, threads)
        line["cpu_baseline"] = {"value": nb / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": f"oracle decode of {len(pairs)} (sequence, head) pairs of {w.name}, "
                                          f"fp64, {dt:.1f} s"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(WORKLOADS) + sorted(EXTRA_WORKLOADS) + sorted(DECODE_WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-configuration records (N = 2K, 8K, 32K, 128K) of the default workload")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.workload in DECODE_WORKLOADS:
        return run_decode(args, DECODE_WORKLOADS[args.workload])
    w = {**WORKLOADS, **EXTRA_WORKLOADS}[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
