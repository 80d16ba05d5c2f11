#!/usr/bin/env python
"""Benchmark: LayerNorm forward + analytical backward on B200 (sm_100a).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One step = one ``ln_forward`` and one ``ln_backward`` call (every step of the
hot path: row statistics, normalise + affine, row gradient sums, dinp, column
partials, fixed-order column finalise) over one batch of the workload
(default: GPT-2 124M LayerNorm, bf16 activations, N = 65536 rows, C = 768).

Metric: compulsory HBM bytes of forward + backward per second (GB/s), with
rows/s and the fraction of the measured HBM copy bandwidth beside it.
Compulsory bytes: forward 2*N*C*s + 8N + 2*C*s, backward 3*N*C*s + 8N + C*s
+ 8C (s = bytes per activation element).

Timing: inputs resident in HBM before the timed region; W untimed warm-up
steps; K timed steps bracketed by a barrier and a device synchronise on both
sides, timed with CUDA events on the launching stream; max over ranks.  L2:
four buffer sets rotate (each 4*N*C*s bytes, 403 MB for the default
workload), and a step's backward reads a set that its forward did not touch,
so no step re-reads an input from the 126 MB L2.

With N > 1 (torchrun, one rank per GPU) every rank processes its own batch
(weak scaling, data-parallel row shards); the path has no exchange step.

``--impl reference`` times the CPU oracle (double precision, the parity
reference) on host cores on a bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "LayerNorm fwd+bwd GB/s and rows/s at 1 B200; % of HBM roofline"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
SETS = 4
EVERY = 64          # per-call events on one timed step in EVERY
# the files that define the kernels and their launch geometry (the ncu
# traffic figure stays valid while these are unchanged)
KERNEL_SOURCES = [os.path.join(ROOT, "layernorm_fwd_bwd_b200", "csrc", f)
                  for f in ("ln_kernels.cuh", "ln_select.cuh", "ln_tma.cuh", "ln_tile.cuh",
                            "ln_split.cuh", "ln_dispatch.cuh", "ln_host.cuh")]
TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "ln_backward_gpt2_124m_bf16.md")


def parse_args():
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20000)
    p.add_argument("--warmup", type=int, default=50)
    p.add_argument("--workload", default="gpt2_124m_bf16")
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--e2e-steps", type=int, default=0,
                   help="end-to-end steps (0: K/500, at least 8)")
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="target CPU time of the oracle baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-variants", action="store_true",
                   help="skip timing ln_forward_residual, ln_backward_ex and fp16")
    p.add_argument("--no-workloads", action="store_true",
                   help="skip timing forward and backward on every workload")
    p.add_argument("--no-loops", action="store_true",
                   help="time the K steps only: no back-to-back call loops, e2e, variants "
                        "or workloads (short runs under a profiler)")
    p.add_argument("--sets", type=int, default=SETS,
                   help="rotating buffer sets (>= 2 so a step's backward never "
                        "reads what its forward just read)")
    return p.parse_args()


def strip_comments(src: str) -> str:
    """C/C++ source without its comments (string and character literals kept
    intact), each line's trailing blanks and blank lines dropped, so that
    editing a comment does not change the hash of the code."""
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
            while i < n and src[i] != "\n":
                i += 1
        elif src.startswith("/*", i):
            end = src.find("*/", i + 2)
            i = n if end < 0 else end + 2
        else:
            out.append(c)
            i += 1
    lines = [line.rstrip() for line in "".join(out).split("\n")]
    return "\n".join(line for line in lines if line)


def source_sha256() -> str:
    """Hash of the kernel sources' code (comments excluded)."""
    h = hashlib.sha256()
    for path in KERNEL_SOURCES:
        with open(path, encoding="utf-8") as f:
            h.update(strip_comments(f.read()).encode())
    return h.hexdigest()


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic():
    """DRAM bytes per ln_backward call from the committed ncu summary, or None
    when it is missing or was taken on different kernel sources."""
    try:
        text = open(TRAFFIC_PROFILE).read()
    except OSError:
        return None
    m = re.search(r"dram_bytes_per_call:\s*(\d+)", text)
    s = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text)
    if not m or not s or s.group(1) != source_sha256():
        return None
    return int(m.group(1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def wait_first_sample(self, timeout: float = 5.0) -> bool:
        """Block until nvidia-smi has written its first line (it needs about
        a second to start), so that samples cover the region that follows."""
        if self.proc is None:
            return False
        t_end = time.time() + timeout
        while time.time() < t_end:
            self.file.flush()
            if os.path.getsize(self.file.name) > 0:
                return True
            if self.proc.poll() is not None:
                return False
            time.sleep(0.05)
        return False

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.file.flush()

    def summary(self, t0: float, t1: float) -> dict:
        self.file.seek(0)
        rows = []
        for line in self.file.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except ValueError:
                continue
        os.unlink(self.file.name)
        inside = [r for r in rows if t0 - 0.25 <= r[0] <= t1 + 0.25]
        if not inside:
            # region shorter than the sampling period: nearest sample(s)
            inside = sorted(rows, key=lambda r: abs(r[0] - 0.5 * (t0 + t1)))[:2]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"],
                    "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[k] for r in inside for k in range(4)
                          if r[3][k].lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside)}


# ------------------------------------------------------------- multi-rank

def max_over_ranks(x: float, device="cpu") -> float:
    """The largest value of x over all ranks (x itself without a process
    group).  Used for every timing: the job is as slow as its slowest rank."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, bytes_per_rank_step: int, step_seconds: float) -> float:
    """Whole-job GB/s: every rank moves bytes_per_rank_step per step (weak
    scaling), and a step takes the slowest rank's time."""
    return world * bytes_per_rank_step / step_seconds / 1e9


# --------------------------------------------------------------------- ours

def run_ours(args, world: int, rank: int, local: int):
    import numpy as np
    import torch
    import torch.distributed as dist

    from layernorm_fwd_bwd_b200 import ln
    from layernorm_fwd_bwd_b200 import workloads as wl

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    w = wl.WORKLOADS[args.workload]
    N, C = w.N, w.C
    tdt = torch.float32 if w.dtype == wl.F32 else torch.bfloat16
    dcode = ln.LN_F32 if w.dtype == wl.F32 else ln.LN_BF16
    batch = wl.generate(w)

    def host_tensor(a):
        if w.dtype == wl.F32:
            return torch.from_numpy(np.ascontiguousarray(a, np.float32))
        return torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).view(
            torch.bfloat16)

    h_inp, h_dout = host_tensor(batch.inp), host_tensor(batch.dout)
    h_w, h_b = host_tensor(batch.weight), host_tensor(batch.bias)
    stream = torch.cuda.Stream(device=dev)
    sp = stream.cuda_stream
    with torch.cuda.stream(stream):
        weight, bias = h_w.to(dev), h_b.to(dev)
        dweight = torch.empty(C, device=dev)
        dbias = torch.empty(C, device=dev)
        sets = []
        nsets = max(2, args.sets)
        for _ in range(nsets):
            sets.append(dict(inp=h_inp.to(dev), dout=h_dout.to(dev),
                             out=torch.empty(N, C, dtype=tdt, device=dev),
                             dinp=torch.empty(N, C, dtype=tdt, device=dev),
                             mean=torch.empty(N, device=dev),
                             rstd=torch.empty(N, device=dev)))
    stream.synchronize()
    eps = batch.eps
    fargs = [(s["out"].data_ptr(), s["mean"].data_ptr(), s["rstd"].data_ptr(),
              s["inp"].data_ptr(), weight.data_ptr(), bias.data_ptr(), N, C, eps,
              dcode, sp) for s in sets]
    bargs = [(s["dinp"].data_ptr(), dweight.data_ptr(), dbias.data_ptr(),
              s["dout"].data_ptr(), s["inp"].data_ptr(), weight.data_ptr(),
              s["mean"].data_ptr(), s["rstd"].data_ptr(), N, C, dcode, sp)
             for s in sets]
    fwd, bwd = ln.raw_forward, ln.raw_backward

    def check(rc):
        if rc != 0:
            raise ln.LNError(rc)

    for k in range(nsets):                      # statistics for every set
        check(fwd(*fargs[k]))

    def step(i, ev=None):
        a, b = i % nsets, (i + nsets // 2) % nsets
        if ev is not None:
            ev[0].record(stream)
        check(fwd(*fargs[a]))
        if ev is not None:
            ev[1].record(stream)
        check(bwd(*bargs[b]))
        if ev is not None:
            ev[2].record(stream)

    K, W = args.steps, args.warmup
    sampler = ClockSampler(local) if rank == 0 else None
    if sampler is not None:
        sampler.wait_first_sample()
    for i in range(W):
        step(i)
    # per-call events on every EVERY-th timed step only: an event record
    # between two launches costs about a microsecond of GPU time and breaks
    # the overlap that programmatic dependent launch gives the finalise
    sampled = [i for i in range(K) if i % EVERY == 0]
    events = {i: [torch.cuda.Event(enable_timing=True) for _ in range(3)] for i in sampled}
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = ln.launch_count()
    t0 = time.time()
    start.record(stream)
    for i in range(K):
        step(W + i, events.get(i))
    end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    if world > 1:
        dist.barrier()
    launches = ln.launch_count() - launches0
    total_ms = start.elapsed_time(end)
    fwd_ms = statistics.fmean(e[0].elapsed_time(e[1]) for e in events.values())
    bwd_ms = statistics.fmean(e[1].elapsed_time(e[2]) for e in events.values())
    total_ms = max_over_ranks(total_ms, dev)

    # each call on its own, back to back (events around the loop only)
    if args.no_loops:
        args.no_e2e = args.no_variants = args.no_workloads = True
        fwd_loop_us, bwd_loop_us = fwd_ms * 1e3, bwd_ms * 1e3
    else:
        fwd_loop_us = call_loop_us(torch, stream, lambda i: check(fwd(*fargs[i % nsets])))
        bwd_loop_us = call_loop_us(torch, stream, lambda i: check(bwd(*bargs[i % nsets])))

    # end to end through the public API with host buffers (pinned)
    e2e = None if args.no_e2e else run_e2e(args, torch, ln, stream, dev, h_inp, h_dout,
                                           h_w, h_b, N, C, tdt, dcode, eps, world)
    variants = None if args.no_variants else run_variants(
        torch, ln, stream, sets, weight, bias, dweight, dbias, w, eps, dcode)
    t_loops = time.time()
    if sampler is not None:
        sampler.stop()
    del sets, fargs, bargs
    workloads = None if (args.no_workloads or rank != 0) else run_workloads(
        torch, ln, stream, dev, args.sets)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    fb, bb = w.fwd_bytes(), w.bwd_bytes()
    step_s = total_ms / 1e3 / K
    value = job_throughput(world, fb + bb, step_s)
    peak, peak_kind = hbm_peak()
    bwd_gbs = bb / (bwd_loop_us / 1e6) / 1e9
    fwd_gbs = fb / (fwd_loop_us / 1e6) / 1e9
    loop_timing = (f"{LOOP_CALLS} back-to-back calls over the rotating sets" if not args.no_loops
                   else "events around each call of the sampled timed steps (--no-loops)")
    clocks = None
    if sampler:
        clocks = sampler.summary(t0, t_loops)
        clocks["window"] = ("from the first timed step to the end of the variant loops: "
                            "timed steps, fwd/bwd call loops, e2e, variants")
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s",
        "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(total_ms / K, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded SplitMix64/Box-Muller, workload distributions)",
        "config": {"workload": w.name, "description": w.description, "N": N, "C": C,
                   "activations": w.dtype, "stats_and_param_grads": "f32",
                   "eps": eps, "rows_per_gpu": N, "parallelism": f"dp{world} (row shards)",
                   "l2": f"{nsets} rotating buffer sets; each step's backward reads a set "
                         "its forward did not touch; inputs never re-read from L2"},
        "rows_per_s": round(world * N / step_s, 1),
        "pct_hbm_measured": round(value / world / peak * 100, 2) if peak_kind == "measured" else None,
        "pct_hbm_nominal_8tbs": round(value / world / NOMINAL_HBM_GBS * 100, 2),
        "fwd": {"us": round(fwd_loop_us, 3), "GB_s": round(fwd_gbs, 1), "bytes": fb,
                "timing": loop_timing,
                "us_sampled_in_step": round(fwd_ms * 1e3, 3)},
        "bwd": {"us": round(bwd_loop_us, 3), "GB_s": round(bwd_gbs, 1), "bytes": bb,
                "timing": loop_timing,
                "us_sampled_in_step": round(bwd_ms * 1e3, 3)},
        "per_call_sampling": f"events around each call on 1 timed step in {EVERY} "
                             f"({len(events)} steps); an event between two launches "
                             "stops their programmatic overlap, so these read high",
        "roofline": {"bound": "hbm", "kernel": "ln_backward (row pass + column finalise)",
                     "achieved": round(bwd_gbs, 1), "peak": peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": round(bwd_gbs / peak, 4),
                     "traffic": profiled_traffic(),
                     "traffic_note": "DRAM bytes (read + write) during one serialised "
                                     "launch of each of the two kernels under ncu; below the "
                                     "algorithmic bytes because part of dinp is still dirty "
                                     "in L2 when a launch ends"},
        "gpu_launches": launches,
        "clocks": clocks,
        "e2e": e2e,
        "variants": variants,
        "workloads": workloads,
    }
    line["cpu_baseline"] = (None if (world > 1 or args.no_cpu_baseline)
                            else cpu_baseline(w, args.cpu_seconds))
    return line


LOOP_CALLS = 500


def call_loop_us(torch, stream, call, calls: int = LOOP_CALLS) -> float:
    """Mean duration of one call in a loop of back-to-back calls, timed with
    CUDA events on the launching stream around the whole loop (after 8
    untimed calls)."""
    for i in range(8):
        call(i)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(calls):
        call(i)
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end) * 1e3 / calls


def graph_loop_us(torch, stream, call, calls: int = 200, reps: int = 3) -> float:
    """Mean duration of one call when `calls` back-to-back calls are captured
    in one CUDA graph on `stream` and the graph is replayed there (median of
    `reps` replays, each timed with CUDA events on that stream, after one
    untimed replay)."""
    for i in range(4):
        call(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(calls):
            call(i)
    times = []
    with torch.cuda.stream(stream):
        g.replay()
        torch.cuda.synchronize()
        for _ in range(reps):
            start = torch.cuda.Event(enable_timing=True)
            end = torch.cuda.Event(enable_timing=True)
            start.record(stream)
            g.replay()
            end.record(stream)
            torch.cuda.synchronize()
            times.append(start.elapsed_time(end) * 1e3 / calls)
    del g
    return sorted(times)[len(times) // 2]


def variant_bytes(w) -> dict:
    """Compulsory HBM bytes of one call of each variant (s = element size):
    residual forward reads resid and branch and writes resid_out and out
    (4NCs) plus the statistics and parameters; accumulating backward also
    reads the previous dinp (4NCs) and reads and writes dweight/dbias;
    recomputing backward skips the 8N bytes of saved statistics."""
    N, C, s = w.N, w.C, w.elem_bytes
    return {"fwd_residual": 4 * N * C * s + 8 * N + 2 * C * s,
            "bwd_accumulate": 4 * N * C * s + 8 * N + C * s + 16 * C,
            "bwd_recompute": 3 * N * C * s + C * s + 8 * C,
            "bwd_accumulate_recompute": 4 * N * C * s + C * s + 16 * C}


def run_variants(torch, ln, stream, sets, weight, bias, dweight, dbias, w, eps, dcode,
                 calls: int = 400) -> dict:
    """Each variant on its own: `calls` calls over the rotating buffer sets
    (inputs never re-read from L2), timed with CUDA events around the loop on
    the launching stream.  The inputs reuse the sets' arrays (a branch is
    another set's dout; accumulation goes into whatever dinp holds), which
    changes no byte counts.  For a 16-bit workload, plain forward and
    backward also run on fp16 copies of the sets."""
    N, C = w.N, w.C
    n = len(sets)
    sp = stream.cuda_stream
    ptr = lambda t: t.data_ptr()
    acc = ln.LN_BWD_ACCUMULATE_DINP | ln.LN_BWD_ACCUMULATE_DPARAMS
    rec = ln.LN_BWD_RECOMPUTE_STATS

    def fwd_res(i):
        a, o = sets[i % n], sets[(i + 1) % n]
        return ln.raw_forward_residual(ptr(a["dinp"]), ptr(a["out"]), ptr(a["mean"]),
                                       ptr(a["rstd"]), ptr(a["inp"]), ptr(o["dout"]),
                                       ptr(weight), ptr(bias), N, C, eps, dcode, sp)

    def bwd_ex(flags):
        def call(i):
            b = sets[i % n]
            st = (None, None) if flags & rec else (ptr(b["mean"]), ptr(b["rstd"]))
            return ln.raw_backward_ex(ptr(b["dinp"]), ptr(dweight), ptr(dbias), ptr(b["dout"]),
                                      ptr(b["inp"]), ptr(weight), st[0], st[1], N, C, eps,
                                      dcode, flags, sp)
        return call

    peak, _ = hbm_peak()
    nbytes = variant_bytes(w)
    out = {}
    def checked(call):
        def run(i):
            rc = call(i)
            if rc != 0:
                raise ln.LNError(rc)
        return run

    cases = [("fwd_residual", fwd_res), ("bwd_accumulate", bwd_ex(acc)),
             ("bwd_recompute", bwd_ex(rec)), ("bwd_accumulate_recompute", bwd_ex(acc | rec))]
    if w.elem_bytes == 2:
        # the same shape with fp16 activations (the sets' values converted)
        with torch.cuda.stream(stream):
            h = [{k: (v.to(torch.float16) if v.dtype == torch.bfloat16 else torch.empty_like(v))
                  for k, v in st.items()} for st in sets]
            hw, hb = weight.to(torch.float16), bias.to(torch.float16)
        f16 = ln.LN_F16

        def h_fwd(i):
            a = h[i % n]
            return ln.raw_forward(ptr(a["out"]), ptr(a["mean"]), ptr(a["rstd"]), ptr(a["inp"]),
                                  ptr(hw), ptr(hb), N, C, eps, f16, sp)

        def h_bwd(i):
            b = h[i % n]
            return ln.raw_backward(ptr(b["dinp"]), ptr(dweight), ptr(dbias), ptr(b["dout"]),
                                   ptr(b["inp"]), ptr(hw), ptr(b["mean"]), ptr(b["rstd"]), N, C,
                                   f16, sp)

        for k in range(n):                  # statistics for every fp16 set
            checked(h_fwd)(k)
        nbytes["fp16_fwd"], nbytes["fp16_bwd"] = w.fwd_bytes(), w.bwd_bytes()
        cases += [("fp16_fwd", h_fwd), ("fp16_bwd", h_bwd)]
    for name, call in cases:
        us = call_loop_us(torch, stream, checked(call), calls)
        gbs = nbytes[name] / (us * 1e-6) / 1e9
        out[name] = {"us": round(us, 3), "GB_s": round(gbs, 1), "bytes": nbytes[name],
                     "frac": round(gbs / peak, 4), "calls": calls}
    return out


def run_workloads(torch, ln, stream, dev, nsets: int, calls: int = LOOP_CALLS) -> dict:
    """ln_forward and ln_backward on every workload at its full size, timed
    like the headline: `calls` back-to-back calls over rotating buffer sets
    (a backward reads a set whose forward ran ``nsets // 2`` calls earlier),
    CUDA events around the loop on the launching stream.  ``fwd_us`` and
    ``bwd_us`` time loops of one call kind, and ``GB_s``, ``frac`` and
    ``rows_per_s`` are fwd+bwd as bytes / (t_fwd + t_bwd).  ``step_us`` times
    the step itself, forward and backward alternating as in the headline's
    timed region (``step_GB_s``, ``step_frac``); ``graph_step_us`` is the
    same step loop captured in one CUDA graph and replayed (the library's
    calls are capturable), which removes the host's launch path but not the
    kernels' own boundaries.  GB/s counts compulsory bytes; fractions are
    against the measured HBM copy bandwidth (or the fallback, as
    ``peak_kind`` says)."""
    import numpy as np

    from layernorm_fwd_bwd_b200 import workloads as wl
    peak, _ = hbm_peak()
    nsets = max(2, nsets)
    out = {}
    for name, w in wl.WORKLOADS.items():
        batch = wl.generate(w)
        N, C = w.N, w.C
        tdt = torch.float32 if w.dtype == wl.F32 else torch.bfloat16
        code = ln.LN_F32 if w.dtype == wl.F32 else ln.LN_BF16

        def dev_t(a):
            if w.dtype == wl.F32:
                t = torch.from_numpy(np.ascontiguousarray(a, np.float32))
            else:
                t = torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).view(
                    torch.bfloat16)
            return t.to(dev, non_blocking=False)

        with torch.cuda.stream(stream):
            inp, dout = dev_t(batch.inp), dev_t(batch.dout)
            weight, bias = dev_t(batch.weight), dev_t(batch.bias)
            dweight, dbias = torch.empty(C, device=dev), torch.empty(C, device=dev)
            sets = [dict(inp=inp.clone(), dout=dout.clone(),
                         out=torch.empty(N, C, dtype=tdt, device=dev),
                         dinp=torch.empty(N, C, dtype=tdt, device=dev),
                         mean=torch.empty(N, device=dev), rstd=torch.empty(N, device=dev))
                    for _ in range(nsets)]
        del inp, dout, batch
        stream.synchronize()
        sp = stream.cuda_stream
        p = lambda t: t.data_ptr()

        def fwd(i):
            a = sets[i % nsets]
            rc = ln.raw_forward(p(a["out"]), p(a["mean"]), p(a["rstd"]), p(a["inp"]),
                                p(weight), p(bias), N, C, 1e-5, code, sp)
            if rc:
                raise ln.LNError(rc)

        def bwd(i):
            b = sets[(i + nsets // 2) % nsets]
            rc = ln.raw_backward(p(b["dinp"]), p(dweight), p(dbias), p(b["dout"]),
                                 p(b["inp"]), p(weight), p(b["mean"]), p(b["rstd"]), N, C,
                                 code, sp)
            if rc:
                raise ln.LNError(rc)

        def step(i):
            fwd(i)
            bwd(i)

        for k in range(nsets):
            fwd(k)
        f_us = call_loop_us(torch, stream, fwd, calls)
        b_us = call_loop_us(torch, stream, bwd, calls)
        s_us = call_loop_us(torch, stream, step, calls)
        g_us = graph_loop_us(torch, stream, step)
        fb, bb = w.fwd_bytes(), w.bwd_bytes()
        sum_gbs = (fb + bb) / ((f_us + b_us) * 1e-6) / 1e9
        step_gbs = (fb + bb) / (s_us * 1e-6) / 1e9
        graph_gbs = (fb + bb) / (g_us * 1e-6) / 1e9
        out[name] = {
            "N": N, "C": C, "dtype": w.dtype,
            "fwd_us": round(f_us, 3), "bwd_us": round(b_us, 3),
            "fwd_GB_s": round(fb / (f_us * 1e-6) / 1e9, 1),
            "bwd_GB_s": round(bb / (b_us * 1e-6) / 1e9, 1),
            "GB_s": round(sum_gbs, 1), "rows_per_s": round(N / ((f_us + b_us) * 1e-6), 1),
            "frac": round(sum_gbs / peak, 4),
            "bwd_frac": round(bb / (b_us * 1e-6) / 1e9 / peak, 4),
            "step_us": round(s_us, 3), "step_GB_s": round(step_gbs, 1),
            "step_frac": round(step_gbs / peak, 4),
            "graph_step_us": round(g_us, 3), "graph_GB_s": round(graph_gbs, 1),
            "graph_frac": round(graph_gbs / peak, 4),
            "bytes": fb + bb,
            "l2": ("inputs smaller than L2: launch-bound correctness case"
                   if nsets * 2 * N * C * w.elem_bytes < 126e6 else
                   f"{nsets} rotating sets, inputs never re-read from L2")}
        del sets
        torch.cuda.empty_cache()
    return out


def run_e2e(args, torch, ln, stream, dev, h_inp, h_dout, h_w, h_b, N, C, tdt, dcode,
            eps, world):
    """Same metric through the public API with host buffers: every step copies
    its inputs from pinned host memory, runs forward and backward, and reads
    every result back into pinned host memory.  Steps are double-buffered the
    way a caller would pipeline them: step i+1's uploads (own stream) overlap
    step i's downloads (own stream) and kernels, so both PCIe directions are
    busy at once; events order each device buffer set's upload after its
    previous download, its kernels after its upload, and its download after
    its kernels."""
    steps = args.e2e_steps or max(8, args.steps // 500)
    pin = {k: v.pin_memory() for k, v in
           dict(inp=h_inp, dout=h_dout, w=h_w, b=h_b).items()}
    out_shapes = dict(out=((N, C), tdt), dinp=((N, C), tdt), mean=((N,), torch.float32),
                      rstd=((N,), torch.float32), dw=((C,), torch.float32),
                      db=((C,), torch.float32))
    hout = [{k: torch.empty(shape, dtype=dt).pin_memory() for k, (shape, dt) in
             out_shapes.items()} for _ in range(2)]
    up = torch.cuda.Stream(device=dev)
    down = torch.cuda.Stream(device=dev)
    d = []
    for _ in range(2):
        with torch.cuda.stream(stream):
            d.append(dict(inp=torch.empty(N, C, dtype=tdt, device=dev),
                          dout=torch.empty(N, C, dtype=tdt, device=dev),
                          w=torch.empty(C, dtype=tdt, device=dev),
                          b=torch.empty(C, dtype=tdt, device=dev),
                          out=torch.empty(N, C, dtype=tdt, device=dev),
                          dinp=torch.empty(N, C, dtype=tdt, device=dev),
                          mean=torch.empty(N, device=dev), rstd=torch.empty(N, device=dev),
                          dw=torch.empty(C, device=dev), db=torch.empty(C, device=dev)))
    torch.cuda.synchronize()
    freed = [None, None]          # event: set k's last download finished

    def one(i):
        k = i % 2
        s = d[k]
        loaded = torch.cuda.Event()
        computed = torch.cuda.Event()
        with torch.cuda.stream(up):
            if freed[k] is not None:
                up.wait_event(freed[k])
            for name in ("inp", "dout", "w", "b"):
                s[name].copy_(pin[name], non_blocking=True)
            loaded.record(up)
        stream.wait_event(loaded)
        ln.ln_forward(s["out"], s["mean"], s["rstd"], s["inp"], s["w"], s["b"], N, C, eps,
                      dcode, stream)
        ln.ln_backward(s["dinp"], s["dw"], s["db"], s["dout"], s["inp"], s["w"], s["mean"],
                       s["rstd"], N, C, dcode, stream)
        computed.record(stream)
        with torch.cuda.stream(down):
            down.wait_event(computed)
            for name in out_shapes:
                hout[k][name].copy_(s[name], non_blocking=True)
            freed[k] = torch.cuda.Event()
            freed[k].record(down)

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    freed[0] = freed[1] = None
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    start.record(up)
    for i in range(steps):
        one(i)
    end.record(down)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(end), dev)
    from layernorm_fwd_bwd_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = sum(v.numel() * v.element_size() for v in hout[0].values())
    step_s = ms / 1e3 / steps
    return {"value": round(job_throughput(world, w.fwd_bytes() + w.bwd_bytes(), step_s), 2),
            "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": steps, "ms_per_step": round(ms / steps, 4),
            "pipelining": "2 buffer sets; uploads, kernels and downloads on 3 streams"}


# ----------------------------------------------------------------- oracle

def _oracle_rate(w, rows_sample: int, seconds: float):
    """Time the CPU oracle (as it stands) on a row sample: forward then
    backward.  Returns (GB/s of compulsory bytes, seconds per pass, passes)."""
    import numpy as np

    import oracle
    from layernorm_fwd_bwd_b200 import workloads as wl
    rows = np.arange(rows_sample, dtype=np.int64)
    b = wl.generate(w, rows=rows)
    x, dy = b.f64("inp"), b.f64("dout")
    wt, bs = b.f64("weight"), b.f64("bias")
    orc = oracle.default()
    times = []
    t_end = time.perf_counter() + seconds
    while True:
        t = time.perf_counter()
        _, m, r = orc.forward(x, wt, bs, b.eps)
        orc.backward(dy, x, wt, m, r)
        times.append(time.perf_counter() - t)
        if time.perf_counter() >= t_end and len(times) >= 1:
            break
    s = w.elem_bytes
    n = rows_sample
    byts = (2 * n * w.C * s + 8 * n + 2 * w.C * s) + (3 * n * w.C * s + 8 * n + w.C * s + 8 * w.C)
    per = statistics.median(times)
    return byts / per / 1e9, per, len(times)


def cpu_baseline(w, seconds: float) -> dict:
    rows = min(w.N, 16384)
    gbs, per, reps = _oracle_rate(w, rows, seconds)
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "host_cores": os.cpu_count(),
            "sample": f"first {rows} of {w.N} rows of {w.name}, forward+backward in "
                      f"double, median of {reps} passes ({per:.3f} s each), "
                      "single thread"}


def run_reference(args, world: int, rank: int):
    """The CPU oracle timed as the reference arm: each step is forward +
    backward over a bounded row sample of the same workload."""
    if rank != 0:
        return None
    from layernorm_fwd_bwd_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    # calibrate: rows per second of the oracle on a small sample
    cal = min(512, w.N)
    _, per, _ = _oracle_rate(w, cal, 0.0)
    rows_per_s = cal / per
    budget = 150.0
    rows = int(max(1, min(w.N, rows_per_s * budget / max(1, args.steps + args.warmup))))
    import numpy as np

    import oracle
    b = wl.generate(w, rows=np.arange(rows, dtype=np.int64))
    x, dy = b.f64("inp"), b.f64("dout")
    wt, bs = b.f64("weight"), b.f64("bias")
    orc = oracle.default()
    for _ in range(args.warmup):
        _, m, r = orc.forward(x, wt, bs, b.eps)
        orc.backward(dy, x, wt, m, r)
    t = time.perf_counter()
    for _ in range(args.steps):
        _, m, r = orc.forward(x, wt, bs, b.eps)
        orc.backward(dy, x, wt, m, r)
    el = time.perf_counter() - t
    s = w.elem_bytes
    byts = (2 * rows * w.C * s + 8 * rows + 2 * w.C * s) + \
        (3 * rows * w.C * s + 8 * rows + w.C * s + 8 * w.C)
    value = byts * args.steps / el / 1e9
    sample = (f"first {rows} of {w.N} rows of {w.name} per step, forward+backward in "
              "double, single thread")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded SplitMix64/Box-Muller, workload distributions)",
        "config": {"workload": w.name, "description": w.description, "N": w.N, "C": w.C,
                   "activations": w.dtype, "rows_per_step_sample": rows},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1,
                         "host_cores": os.cpu_count(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and not (world == 1 and args.gpus == 1):
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE",
              file=sys.stderr)
    if args.impl == "reference":
        line = run_reference(args, world, rank)
    else:
        line = run_ours(args, world, rank, local)
    if line is not None and rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
