"""Benchmark of the KLA hot path on B200: prefill tokens/s (+ roofline) and
decode tokens/s (+ HBM GB/s), one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill_4k]
  python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N
  python bench.py --impl reference     # the fp64 oracle on the host cores

A step is one prefill of the workload (default: the 0.4B-scale layer,
B=8 T=4096 H=8 d=128, bf16) through kla_chunk_fwd.  Each rank processes its
own batch (independent sequences, no collective on the data path): weak
scaling.  L2 is flushed (512 MiB written then read) before every timed step
and each step is bracketed by CUDA events on the launching stream; the job
time is the max over ranks.  The other halves of the prefill metric (65K
context, the stress shape) are timed the same way and reported under
"other_workloads".  The decode workload (B=64 H=16 d=128, 32K-token state)
is timed as 1000 consecutive in-place steps with one event pair, on one
state and on a rotating set of three states larger than L2, and reported
under "decode".
"""
from __future__ import annotations

import argparse
import functools
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# --------------------------------------------------------------- workloads
def prefill_work(w):
    """Algorithmic flops and minimum HBM bytes of one whole prefill: q, k, v
    read and o written once, g and eta read once, h0 read (when given) and
    h_T written.  Dense tensor work per head-token: five (C x C x d) products
    (K K^T, Q K^T, T'' K, T' V, P V') and three (C x d x d) ones (W h, Q h,
    K^T V')."""
    C = 64
    d = w.dk
    es = 2 if w.dtype == "bf16" else 4
    ntok = w.B * w.T * w.H  # head-tokens
    flops = ntok * (10 * C * d + 6 * d * d)
    state = w.B * w.H * w.dk * w.dv * 4
    byts = ntok * (2 * w.dk + 2 * w.dv) * es + ntok * 8 + state * (2 if w.kind == "stress" else 1)
    return flops, byts


def stage_work(w):
    """Algorithmic flops and bytes of each of the two kernels of one prefill
    (minimum bytes: the inputs a kernel must read and the
    outputs it must write; the per-chunk factors T', T'' that the first
    kernel hands the second are an intermediate of this split, not
    algorithmic bytes, and are reported separately).

    UT transform: reads k, g, eta; flops of K K^T.  State/output kernel:
    reads q, k, v, g (and h0); writes o and h_T; flops of the other seven
    products."""
    C = 64
    d = w.dk
    es = 2
    ntok = w.B * w.T * w.H
    nchunk = w.B * w.H * ((w.T + C - 1) // C)
    fac = nchunk * 2 * C * C * 2
    state = w.B * w.H * w.dk * w.dv * 4
    ut = {"flops": ntok * 2 * C * d, "bytes": ntok * w.dk * es + ntok * 8,
          "intermediate_bytes": fac}
    chain = {"flops": ntok * (8 * C * d + 6 * d * d),
             "bytes": ntok * (2 * w.dk + 2 * w.dv) * es + ntok * 4
             + state * (2 if w.kind == "stress" else 1),
             "intermediate_bytes": fac}
    return ut, chain


def profiled_traffic(kernel_file, profile):
    """DRAM bytes per launch recorded by an ncu capture summarised under
    profiles/, if the kernel source is unchanged since (same sha256)."""
    import hashlib
    src = os.path.join(ROOT, "delta_rule_linear_kla_b200", "csrc", kernel_file)
    prof = os.path.join(ROOT, "profiles", profile)
    if not (os.path.exists(src) and os.path.exists(prof)):
        return None
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    rec = {}
    for line in open(prof):
        if ":" in line and line.startswith(("source-sha256", "dram-bytes-per-launch")):
            k, v = line.split(":", 1)
            rec[k.strip()] = v.strip()
    if rec.get("source-sha256") != digest:
        return None
    try:
        return int(rec["dram-bytes-per-launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason sampling during a timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.perf_counter(), [c.strip() for c in line.split(",")]))

    def wait_first(self, timeout=3.0):
        t0 = time.perf_counter()
        while self.proc and not self.rows and time.perf_counter() - t0 < timeout:
            time.sleep(0.02)

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t_lo=None, t_hi=None):
        """Median SM clock (upper half of the samples: under load) and the
        throttle reasons seen between host times t_lo and t_hi."""
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, r in self.rows:
            if (t_lo is not None and ts < t_lo) or (t_hi is not None and ts > t_hi):
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except (ValueError, IndexError):
                continue
            for n, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        busy = sorted(sm)[len(sm) // 2:]  # upper half: samples under load
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


class L2Flush:
    """Writes then reads a buffer larger than L2 (126 MB on B200), so the next
    kernel starts with a cold L2 and no dirty lines to write back."""

    def __init__(self, dev, mib=512):
        self.buf = torch.empty(mib * (1 << 20) // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        self.buf.fill_(1.0)
        self.buf.sum()


def metric_name(workload):
    if workload == "prefill_4k":
        return "prefill tokens/s (0.4B-scale layer, T=4096)"
    return "prefill tokens/s (%s)" % workload


# ------------------------------------------------------------- our arm
def run_ours(args, rank, world, dev):
    from delta_rule_linear_kla_b200 import api, inputs

    peaks, peak_src = load_peaks()
    w = inputs.WORKLOADS[args.workload]
    w = rank_workload(w, rank)
    x = inputs.make_prefill(w)
    xd = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=w.torch_dtype, device=dev)
    hT = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    chunk = args.path == "chunk"
    if chunk:
        nws = api.chunk_fwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype)
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
        fn = functools.partial(api.chunk_fwd, workspace=ws)
        nseg = api.chunk_fwd_segments(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype, nws)
        # one launch (UT lanes and state CTAs together), or the UT kernel
        # then one chain launch, or for a cut chain of S segments S + 1
        # launches after the UT kernel (segment transitions, one start-state
        # launch per segment boundary, outputs)
        single = api.chunk_fwd_single_launch(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype, nws)
        launches_per_step = 1 if single else 1 + (nseg + 1 if nseg > 1 else 1)
    else:
        fn = api.recurrent_fwd
        nseg, launches_per_step, single = 0, 1, False
    stream = torch.cuda.current_stream()
    flush = L2Flush(dev)

    def step(mid=None):
        # the single launch through chunk_fwd; otherwise the chunk path as
        # its two stages, with an event between them when the split is being
        # timed.  For an uncut chain that is exactly what chunk_fwd launches.
        # For a cut chain chunk_fwd makes the last segment's factors beside
        # the first chain pass instead of before it, so this step (factors of
        # every chunk, then the cut chain) is the staged form; the 65K entry
        # of "other_workloads" times chunk_fwd itself
        if single:
            fn(xd["q"], xd["k"], xd["v"], xd["g"], xd["eta"], x["eps"], xd["h0"], o=o, hT=hT)
        elif chunk:
            api.chunk_ut_transform(xd["k"], xd["g"], xd["eta"], x["eps"], workspace=ws)
            if mid is not None:
                mid.record(stream)
            api.chunk_state_fwd(xd["q"], xd["k"], xd["v"], xd["g"], ws, xd["h0"], o=o, hT=hT)
        else:
            fn(xd["q"], xd["k"], xd["v"], xd["g"], xd["eta"], x["eps"], xd["h0"], o=o, hT=hT)

    clk = ClockSampler(dev.index).__enter__()
    clk.wait_first()
    # warm-up: at least W steps, and at least ~1 s of back-to-back steps so
    # the clock samples that bracket the timed region are taken under load
    t_load = time.perf_counter()
    i = 0
    while i < args.warmup or time.perf_counter() - t_load < args.min_warmup_s:
        flush()
        step()
        i += 1
        if i % 8 == 0:
            torch.cuda.synchronize()
    api.check_device_error()
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3))
           for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for e0, em, e1 in evs:
        flush()
        e0.record(stream)
        step(em)
        e1.record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    t1 = time.perf_counter()
    barrier(world)
    api.check_device_error()
    ms = sum(a.elapsed_time(b) for a, _, b in evs) / args.steps
    ms_max = allreduce_max(ms, world, dev)
    # per-kernel launch durations over the same timed steps (two-kernel path)
    two = chunk and not single
    ms_ut = sum(a.elapsed_time(m) for a, m, _ in evs) / args.steps if two else 0.0
    ms_chain = sum(m.elapsed_time(b) for _, m, b in evs) / args.steps if two else ms

    value = aggregate_throughput(w.B * w.T, world, ms_max)
    flops, byts = prefill_work(w)
    achieved_tf = flops / (ms / 1e3) / 1e12
    hbm_peak = float(peaks["hbm_gbs"])
    tc_peak = float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
    if two:
        ut_w, chain_w = stage_work(w)
    else:
        # one kernel does the whole step: its algorithmic bytes and flops are
        # the step's (the per-chunk factors stay in L2 between its CTAs)
        ut_w, chain_w = None, {"flops": flops, "bytes": byts, "intermediate_bytes": None}
    chain_gbs = chain_w["bytes"] / (ms_chain / 1e3) / 1e9
    kernel_name = ("prefill_kernel" if single else "chain_kernel") if chunk else "recurrent_kernel"
    traffic = (profiled_traffic("kla_chunk_tc.cu", "%s_prefill_4k.md" % kernel_name)
               if chunk and w.name == "prefill_4k" else None)

    # end to end through the public API with host buffers (pinned)
    e2e = None if args.no_e2e else measure_e2e(args, w, x, fn, dev, stream, world)

    res = {
        "metric": metric_name(args.workload),
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded PCG64, distributions of the workload recipe)",
        "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv,
                   "chunk": 64, "path": args.path, "chain_segments": nseg,
                   "global_batch": w.B * world,
                   "seq_len": w.T, "parallelism": "dp%d (independent sequences)" % world,
                   "l2": "flushed before every timed step (512 MiB write+read); inputs > L2"},
        # dominant kernel: the state/output (chain) kernel; its bytes at
        # the measured copy bandwidth take longer than its flops at the
        # measured bf16 rate, so it is HBM-bound at the roofline.  Its
        # algorithmic bytes are the inputs it must read and the outputs it
        # must write (q, k, v, g, h0, o, h_T); the per-chunk factors it also
        # reads are an intermediate of the two-kernel split and show up in
        # "traffic" (ncu DRAM bytes per launch) and "traffic_over_algorithmic"
        "roofline": dict({"kernel": kernel_name,
                          "bound": "hbm", "achieved": chain_gbs, "peak": hbm_peak,
                          "unit": "GB/s", "frac": chain_gbs / hbm_peak,
                          "traffic": traffic,
                          "traffic_over_algorithmic": (None if traffic is None
                                                       else traffic / chain_w["bytes"]),
                          "algorithmic_bytes": chain_w["bytes"],
                          "intermediate_bytes_read": chain_w.get("intermediate_bytes"),
                          "us_per_launch": ms_chain * 1e3,
                          "tensor_tflops": chain_w["flops"] / (ms_chain / 1e3) / 1e12,
                          "peak_source": peak_src + " (burst copy)"}),
        # whole step against the dense bf16 tensor peak (tensor-pipe %)
        "tensor": {"achieved": achieved_tf, "peak": tc_peak, "unit": "TFLOP/s",
                   "frac": achieved_tf / tc_peak, "algorithmic_flops": flops,
                   "algorithmic_bytes": byts,
                   "hbm_frac": byts / (ms / 1e3) / 1e9 / hbm_peak,
                   "peak_source": peak_src + " (burst cuBLAS bf16)"},
        # our kernels per step: one single-launch prefill, or UT transform +
        # chain (S + 1 launches for a chain cut into S segments), one token-serial
        # kernel otherwise; the L2 flush and the flag clear are not counted
        "gpu_launches": args.steps * launches_per_step,
        "wall_s": wall,
        "e2e": e2e,
    }
    if single:
        res["kernels"] = {
            "prefill_kernel": {"us_per_launch": ms * 1e3, "algorithmic_bytes": byts,
                               "gbs": byts / (ms / 1e3) / 1e9,
                               "tflops": flops / (ms / 1e3) / 1e12,
                               "launch": "cooperative, one CTA per SM: %d state CTAs and UT "
                                         "lanes on the other SMs" % (w.B * w.H * w.dv // 64),
                               "note": "event time of the step (the kernel and the clear of "
                                       "its chunk flags)"}}
    elif chunk:
        res["kernels"] = {
            "ut_kernel": {"us_per_launch": ms_ut * 1e3, "algorithmic_bytes": ut_w["bytes"],
                          "gbs": ut_w["bytes"] / (ms_ut / 1e3) / 1e9,
                          "tflops": ut_w["flops"] / (ms_ut / 1e3) / 1e12},
            "chain_kernel": {"us_per_launch": ms_chain * 1e3,
                             "algorithmic_bytes": chain_w["bytes"], "gbs": chain_gbs,
                             "tflops": chain_w["flops"] / (ms_chain / 1e3) / 1e12}}
        if nseg > 1:
            # the cut chain: its time spans its S + 1 launches
            res["kernels"]["chain_kernel"]["launches"] = (
                "%d segments: transitions, start states, outputs" % nseg)
    if chunk and not args.no_other and args.workload == "prefill_4k":
        # the other halves of the prefill metric: 65K context and the
        # stress shape, each its own workload through the same entry point
        res["other_workloads"] = {
            name: time_prefill(inputs.WORKLOADS[name], dev, stream, flush, peaks, rank)
            for name in ("prefill_65k", "stress")}
    if not args.no_decode:
        res["decode"] = run_decode(args, rank, dev, stream, peaks, peak_src, fn, clk)
    if not args.no_kda and w.dtype == "bf16":
        res["kda_prefill"] = run_kda_prefill(w, dev, stream, flush, peaks, peak_src)
    if not args.no_bwd:
        res["backward"] = run_backward(w, dev, stream, flush, peaks, peak_src)
    time.sleep(0.25)
    clk.__exit__()
    res["clocks"] = clk.summary(t_load, t1 + 0.15)
    res["clocks"]["window"] = "samples from 1 s of back-to-back warm-up steps and the timed steps"
    res["warmup_steps_run"] = i
    return res


def time_prefill(w, dev, stream, flush, peaks, rank, steps=5, warmup=3):
    """One more prefill workload through kla_chunk_fwd (workspace allocated
    once, L2 flushed before every step, CUDA events per step): tokens/s and
    its fractions of the measured tensor and HBM peaks on the algorithmic
    flops and bytes."""
    from delta_rule_linear_kla_b200 import api

    w = rank_workload(w, rank)
    x = inputs_to(dev, w)
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=w.torch_dtype, device=dev)
    hT = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    nws = api.chunk_fwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
    nseg = api.chunk_fwd_segments(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype, nws)
    run = lambda: api.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"],
                                o=o, hT=hT, workspace=ws)
    for _ in range(warmup):
        flush()
        run()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    torch.cuda.synchronize()
    for e0, e1 in evs:
        flush()
        e0.record(stream)
        run()
        e1.record(stream)
    torch.cuda.synchronize()
    api.check_device_error()
    ms = sum(a.elapsed_time(b) for a, b in evs) / steps
    flops, byts = prefill_work(w)
    tf = flops / (ms / 1e3) / 1e12
    return {"metric": metric_name(w.name), "value": w.B * w.T / (ms / 1e3),
            "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk,
                       "dv": w.dv, "chain_segments": nseg},
            "tensor": {"achieved": tf, "unit": "TFLOP/s",
                       "frac": tf / float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])),
                       "algorithmic_flops": flops},
            "hbm": {"achieved": byts / (ms / 1e3) / 1e9, "unit": "GB/s",
                    "frac": byts / (ms / 1e3) / 1e9 / float(peaks["hbm_gbs"]),
                    "algorithmic_bytes": byts},
            "l2": "flushed before every timed step"}


def inputs_to(dev, w):
    from delta_rule_linear_kla_b200 import inputs

    x = inputs.make_prefill(w)
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def measure_e2e(args, w, x, fn, dev, stream, world):
    """Same metric end to end from pinned host buffers: H2D of the step's
    inputs, the prefill, D2H of o and hT, all inside the events.  The chunk
    path goes through the C ABI's host-buffer entry point
    (kla_chunk_fwd_host), which pipelines the copies against the kernels
    sequence by sequence; the token-serial path copies, runs and copies back
    in turn."""
    from delta_rule_linear_kla_b200 import api

    host = {k: x[k].pin_memory() for k in ("q", "k", "v", "g", "eta")}
    o_h = torch.empty((w.B, w.T, w.H, w.dv), dtype=w.torch_dtype).pin_memory()
    h_h = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_h.numel() * o_h.element_size() + h_h.numel() * h_h.element_size()
    if args.path == "chunk":
        need = api.chunk_fwd_host_staging_size(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype)
        staging = torch.empty(need, dtype=torch.uint8, device=dev)

        def step():
            api.chunk_fwd_host(host["q"], host["k"], host["v"], host["g"], host["eta"],
                               x["eps"], None, o=o_h, hT=h_h, staging=staging, stream=stream)
        how = "kla_chunk_fwd_host (copies pipelined per sequence against the kernels)"
    else:
        dbuf = {k: torch.empty_like(host[k], device=dev) for k in host}
        o = torch.empty_like(o_h, device=dev)
        hT = torch.empty_like(h_h, device=dev)

        def step():
            for k in dbuf:
                dbuf[k].copy_(host[k], non_blocking=True)
            fn(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["g"], dbuf["eta"], x["eps"], None, o=o,
               hT=hT)
            o_h.copy_(o, non_blocking=True)
            h_h.copy_(hT, non_blocking=True)
        how = "H2D copies, kla_recurrent_fwd, D2H copies in turn"
    n = max(2, min(args.steps, 5))
    times = []
    for i in range(n + 2):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= 2:
            times.append(e0.elapsed_time(e1))
    ms = allreduce_max(sum(times) / len(times), world, dev)
    return {"value": w.B * w.T * world / (ms / 1e3), "unit": "tokens/s",
            "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "path": how}


def _timed_steps(stream, nsteps, body):
    """Times ``nsteps`` back-to-back calls ``body(i)`` with one CUDA event
    pair on ``stream`` (no flush or sync between steps); ms per step."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(nsteps):
        body(i)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / nsteps


def run_decode(args, rank, dev, stream, peaks, peak_src, prefill_fn, clk):
    """Decode: state = our prefill over the trailing prefix; then in-place
    steps, 1000 consecutive ones timed with one event pair.

    Two timings.  "value": every step updates the same 64 MiB state in
    place, exactly the workload as stated; the state fits in the 126 MB L2,
    so part of its traffic never reaches DRAM.  "roofline": the same steps
    on a rotating set of three states (three batches of 64 sequences,
    192 MiB > L2), step i on state i % 3, so every step's read and its
    write-back of the previous steps' dirty lines go through HBM inside
    the timed window; the HBM fraction is taken from this one."""
    from delta_rule_linear_kla_b200 import api, inputs

    w = inputs.DECODE.scaled(seed=inputs.DECODE.seed + 100 * rank)
    nsteps = args.decode_steps
    d = inputs.make_decode(w, steps=nsteps)
    p = {k: v.to(dev) for k, v in d["prefix"].items()}
    _, S = prefill_fn(p["q"], p["k"], p["v"], p["g"], p["eta"], d["eps"], None)
    st = {k: v.to(dev) for k, v in d["steps"].items()}
    o = torch.empty((w.B, w.H, w.dv), dtype=w.torch_dtype, device=dev)
    states = [S] + [S.clone() for _ in range(2)]

    def step(i, S_i):
        api.decode_step(st["q"][i], st["k"][i], st["v"][i], st["g"][i], st["eta"][i], S_i,
                        d["eps"], o=o)

    for i in range(6):
        step(i, states[i % 3])
    t0 = time.perf_counter()
    ms_one = _timed_steps(stream, nsteps, lambda i: step(i, states[0]))
    ms_rot = _timed_steps(stream, nsteps, lambda i: step(i, states[i % 3]))
    t1 = time.perf_counter()
    api.check_device_error()
    state_bytes = 2 * w.B * w.H * w.dk * w.dv * 4
    io_bytes = w.B * w.H * (2 * w.dk + 2 * w.dv) * 2 + w.B * w.H * 8
    gbs = (state_bytes + io_bytes) / (ms_rot / 1e3) / 1e9
    gbs_one = (state_bytes + io_bytes) / (ms_one / 1e3) / 1e9
    peak = float(peaks["hbm_gbs"])

    # the same steps with a per-channel gate (KDA form): 16 gate sets of
    # [B, H, dk] drawn once and cycled (the gate values do not change the
    # work); one more [B, H, dk] fp32 read per step than the scalar gate
    gv = inputs.channel_gates((16, w.B, w.H, w.dk), w.seed + 7).to(dev)

    def kstep(i, S_i):
        api.kda_decode_step(st["q"][i], st["k"][i], st["v"][i], gv[i % 16], st["eta"][i], S_i,
                            d["eps"], o=o)

    for i in range(6):
        kstep(i, states[i % 3])
    kms = _timed_steps(stream, nsteps, lambda i: kstep(i, states[i % 3]))
    api.check_device_error()
    kbytes = state_bytes + io_bytes + w.B * w.H * (w.dk - 1) * 4
    kgbs = kbytes / (kms / 1e3) / 1e9
    return {"metric": "decode tokens/s (B=64 H=16 d=128, 32K-token state)",
            "value": w.B / (ms_one / 1e3), "unit": "tokens/s", "us_per_step": ms_one * 1e3,
            "steps": nsteps,
            "timing": "%d consecutive in-place steps on one state, one event pair, no flush "
                      "(the 64 MiB state stays partly in L2)" % nsteps,
            "rotating_states": {
                "value": w.B / (ms_rot / 1e3), "unit": "tokens/s", "us_per_step": ms_rot * 1e3,
                "timing": "%d consecutive steps over 3 states of 64 MiB (192 MiB > L2), step "
                          "i on state i %% 3, one event pair" % nsteps},
            "clocks": clk.summary(t0, t1 + 0.15), "gpu_launches": 2 * nsteps,
            "roofline": {"kernel": "decode_kernel", "bound": "hbm", "achieved": gbs,
                         "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "timing": "rotating states (every step's bytes cross HBM)",
                         "traffic": profiled_traffic("kla_decode.cu",
                                                     "decode_kernel_decode_b64.md"),
                         "algorithmic_bytes": state_bytes + io_bytes,
                         "one_state_gbs": gbs_one,
                         "peak_source": peak_src},
            "per_channel_gate": {
                "value": w.B / (kms / 1e3), "unit": "tokens/s", "us_per_step": kms * 1e3,
                "steps": nsteps, "gpu_launches": nsteps,
                "timing": "rotating states, as the roofline above",
                "roofline": {"kernel": "decode_kernel (per-channel gate)", "bound": "hbm",
                             "achieved": kgbs, "peak": peak, "unit": "GB/s",
                             "frac": kgbs / peak, "traffic": None,
                             "algorithmic_bytes": kbytes, "peak_source": peak_src}}}


def run_kda_prefill(w, dev, stream, flush, peaks, peak_src, steps=3):
    """The per-channel-gate prefill through kla_kda_chunk_fwd on the same
    workload's q, k, v, eta with per-channel gates: time per call and
    achieved GB/s of its algorithmic bytes (q, k, v, o, the [B,T,H,dk]
    gates, eta, h_T)."""
    from delta_rule_linear_kla_b200 import api, inputs

    x = inputs.make_prefill(w)
    xd = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    gv = inputs.channel_gates((w.B, w.T, w.H, w.dk), w.seed + 11).to(dev)
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=w.torch_dtype, device=dev)
    hT = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, api.kda_chunk_fwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv,
                                                             w.torch_dtype)),
                     dtype=torch.uint8, device=dev)
    run = lambda: api.kda_chunk_fwd(xd["q"], xd["k"], xd["v"], gv, xd["eta"], x["eps"],
                                    xd["h0"], o=o, hT=hT, workspace=ws)
    run()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for e0, e1 in evs:
        flush()
        e0.record(stream)
        run()
        e1.record(stream)
    torch.cuda.synchronize()
    api.check_device_error()
    ms = sum(a.elapsed_time(b) for a, b in evs) / steps
    es = 2 if w.dtype == "bf16" else 4
    ntok = w.B * w.T * w.H
    byts = ntok * (2 * w.dk + 2 * w.dv) * es + ntok * (w.dk + 1) * 4 + w.B * w.H * w.dk * w.dv * 4
    gbs = byts / (ms / 1e3) / 1e9
    peak = float(peaks["hbm_gbs"])
    return {"metric": "prefill tokens/s, per-channel gate (%s)" % w.name,
            "value": w.B * w.T / (ms / 1e3), "unit": "tokens/s", "ms_per_call": ms,
            "calls": steps,
            "path": "kla_kda_chunk_fwd: the token-serial per-channel kernel (the chunk "
                    "kernels of this form are not used: intermittent faults, cause not "
                    "found)",
            "roofline": {"kernel": "whole call", "bound": "hbm",
                         "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "traffic": None, "algorithmic_bytes": byts,
                         "peak_source": peak_src}}


def run_backward(w, dev, stream, flush, peaks, peak_src, steps=2):
    """Gradients of the prefill (chunkwise backward; the token-serial one
    timed beside it) on the same workload for a seeded dL/do and dL/dh_T:
    time per call and achieved GB/s of its algorithmic bytes (reads q, k, v,
    dL/do, g, eta, dL/dh_T; writes the fp32 gradients of q, k, v, g, eta,
    h0)."""
    from delta_rule_linear_kla_b200 import api, inputs

    x = inputs.make_prefill(w)
    xd = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    gen = torch.Generator(device="cpu").manual_seed(w.seed + 21)
    do = torch.randn((w.B, w.T, w.H, w.dv), generator=gen).to(w.torch_dtype).to(dev)
    dhT = torch.randn((w.B, w.H, w.dk, w.dv), generator=gen).to(dev)
    def timed(fn, wsize):
        ws = torch.empty(max(1, wsize), dtype=torch.uint8, device=dev)
        run = lambda: fn(xd["q"], xd["k"], xd["v"], xd["g"], xd["eta"], do, x["eps"],
                         xd["h0"], dhT, workspace=ws, stream=stream)
        run()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for e0, e1 in evs:
            flush()
            e0.record(stream)
            run()
            e1.record(stream)
        torch.cuda.synchronize()
        api.check_device_error()
        del ws
        return sum(a.elapsed_time(b) for a, b in evs) / steps

    ms = timed(api.chunk_bwd, api.chunk_bwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv,
                                                           w.torch_dtype))
    ms_serial = timed(api.recurrent_bwd, api.recurrent_bwd_workspace_size(w.B, w.T, w.H, w.dk,
                                                                          w.dv))
    es = 2 if w.dtype == "bf16" else 4
    ntok = w.B * w.T * w.H
    sb = w.B * w.H * w.dk * w.dv * 4
    byts = (ntok * (2 * w.dk + 2 * w.dv) * es + ntok * 2 * 4 + sb
            + ntok * (2 * w.dk + w.dv + 2) * 4 + sb)
    gbs = byts / (ms / 1e3) / 1e9
    peak = float(peaks["hbm_gbs"])
    return {"metric": "backward tokens/s (%s)" % w.name,
            "value": w.B * w.T / (ms / 1e3), "unit": "tokens/s", "ms_per_call": ms,
            "calls": steps, "dtype": "f32",
            "path": "kla_chunk_bwd: forward chunk prefill writing every chunk-start state, "
                    "cbwd_prep_kernel, cbwd_adjoint_kernel (reverse state-adjoint chain), "
                    "cbwd_grad_kernel (warp-level tf32 tensor-core products)",
            "token_serial_ms_per_call": ms_serial,
            "roofline": {"kernel": "whole call", "bound": "hbm",
                         "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "traffic": None, "algorithmic_bytes": byts,
                         "peak_source": peak_src,
                         "note": "the per-chunk kernels are bound by issuing their "
                                 "warp-level products' operand loads, not by HBM"}}


# ------------------------------------------------------------ reference
def oracle_sample(w, budget_s):
    """Size a sample of workload ``w`` that costs the oracle about
    ``budget_s`` seconds on this host: heads drawn like ``w`` (a multiple of
    the oracle's thread count, up to B*H), length up to T, and whole repeats
    of that when the full workload costs less than the budget."""
    import oracle
    from delta_rule_linear_kla_b200 import inputs

    cores = oracle.num_threads()
    nh_p = min(w.B * w.H, max(cores, 1))
    T_p = min(w.T, 256)
    xp = inputs.make_prefill(w.scaled(B=(nh_p + w.H - 1) // w.H, H=min(w.H, nh_p), T=T_p))
    t0 = time.perf_counter()
    oracle.forward(xp["q"], xp["k"], xp["v"], xp["g"], xp["eta"], xp["eps"], xp["h0"])
    per_round = (time.perf_counter() - t0) / T_p  # s per token for nh_p heads in parallel
    rounds = budget_s / max(per_round, 1e-9)       # affordable token-rounds of nh_p heads
    T_s = int(min(w.T, max(T_p, rounds)))
    groups = max(1, min((w.B * w.H) // nh_p, int(rounds / T_s)))
    nh = min(w.B * w.H, groups * nh_p)
    reps = max(1, min(64, int(rounds / (T_s * groups))))
    H_s = min(w.H, nh)
    B_s = (nh + H_s - 1) // H_s
    xs = inputs.make_prefill(w.scaled(B=B_s, H=H_s, T=T_s))
    return xs, B_s, H_s, T_s, reps, cores


def run_oracle_sample(xs, reps):
    import oracle

    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.forward(xs["q"], xs["k"], xs["v"], xs["g"], xs["eta"], xs["eps"], xs["h0"])
    return time.perf_counter() - t0


def sample_text(w, B_s, H_s, T_s, reps, t):
    return "%d of %d heads x T=%d of %s, drawn with the same distributions, run %d time(s): " \
           "%.1f s of fp64 CPU work" % (B_s * H_s, w.B * w.H, T_s, w.name, reps, t)


def run_reference(args, world, rank):
    """The fp64 oracle on the host cores; each step a bounded sample of the
    workload sized so the whole run stays within a few minutes."""
    from delta_rule_linear_kla_b200 import inputs

    w = inputs.WORKLOADS[args.workload]
    per_step = min(10.0, max(0.5, 100.0 / (args.steps + args.warmup)))
    xs, B_s, H_s, T_s, reps, cores = oracle_sample(w, per_step)
    for _ in range(args.warmup):
        run_oracle_sample(xs, 1)
    times = [run_oracle_sample(xs, reps) for _ in range(args.steps)]
    t = sum(times) / len(times)
    value = B_s * H_s * T_s * reps / w.H / t  # a token = one position of all H heads
    sample = sample_text(w, B_s, H_s, T_s, reps, t) + " per step"
    return {"metric": metric_name(args.workload),
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded PCG64)", "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk,
                       "dv": w.dv, "chunk": 64},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def cpu_baseline(args, budget_s=15.0):
    """The oracle as it stands, timed on this host on a bounded sample."""
    from delta_rule_linear_kla_b200 import inputs

    w = inputs.WORKLOADS[args.workload]
    xs, B_s, H_s, T_s, reps, cores = oracle_sample(w, budget_s)
    t = run_oracle_sample(xs, reps)
    value = B_s * H_s * T_s * reps / w.H / t
    return {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": sample_text(w, B_s, H_s, T_s, reps, t)}


# ---------------------------------------------------------- distributed
def rank_workload(w, rank):
    """Weak scaling: every rank runs its own sequences of the same shape
    (independent heads need no exchange), drawn with a rank-specific seed."""
    return w.scaled(seed=w.seed + 100 * rank)


def aggregate_throughput(units_per_rank, world, ms_max):
    """Whole-job rate: the units all ranks processed over the slowest rank's
    time (ms_max is already the max over ranks)."""
    return units_per_rank * world / (ms_max / 1e3)


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def allreduce_max(x, world, dev):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_4k",
                    choices=["prefill_4k", "prefill_65k", "stress", "tiny"])
    ap.add_argument("--path", choices=["chunk", "recurrent"], default="chunk")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end (host buffers) measurement, e.g. for a "
                         "profiler's launch list of the prefill alone")
    ap.add_argument("--no-kda", action="store_true",
                    help="skip the per-channel-gate (KDA form) prefill measurement")
    ap.add_argument("--no-bwd", action="store_true",
                    help="skip the backward (gradients) measurement")
    ap.add_argument("--min-warmup-s", type=float, default=1.0,
                    help="seconds of back-to-back warm-up steps before timing (clock "
                         "samples under load); 0 for a profiler's short command")
    ap.add_argument("--no-other", action="store_true",
                    help="skip the 65K and stress prefill workloads")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the decode measurement (e.g. under a profiler) and print "
                         "its JSON object")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, world, rank)), flush=True)
        return 0

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", device_id=dev,
                                             timeout=datetime.timedelta(seconds=120))
    if args.decode_only:
        from delta_rule_linear_kla_b200 import api
        peaks, peak_src = load_peaks()
        clk = ClockSampler(dev.index).__enter__()
        res = run_decode(args, rank, dev, torch.cuda.current_stream(), peaks, peak_src,
                         api.chunk_fwd, clk)
        clk.__exit__()
        if rank == 0:
            print(json.dumps(res), flush=True)
        return 0
    try:
        res = run_ours(args, rank, world, dev)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(args)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
