"""Run by test_parity_gpu.test_concurrent_host_threads in a fresh process:
several host threads call the library at once, each on its own stream, before
any other call in the process, so that the per-device set-up (SM count,
workspace pool), the per-kernel shared-memory limits and the occupancy cache
are all filled concurrently.  Then the same calls run again from one thread
on one stream, and every output must match the threaded run bit for bit (the
library's results are deterministic).  Prints one JSON line.  No LayerNorm
arithmetic here: both runs are the library's."""
from __future__ import annotations

import json
import os
import sys
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

from gpu_util import DT, TORCH_DT, bits, to_device  # noqa: E402
from layernorm_fwd_bwd_b200 import ln  # noqa: E402
from layernorm_fwd_bwd_b200 import workloads as wl  # noqa: E402

# (dtype, N, C): widths that reach different kernels (one-warp tile and
# ring, two-warp forward tile with a shared-row ring, the split backward,
# fp32 rings), each with its own shared-memory size
SHAPES = [("bf16", 3001, 1368), ("bf16", 1203, 2456), ("f16", 2047, 1800),
          ("f32", 1500, 1004), ("bf16", 4100, 776), ("f32", 777, 2600)]
REPEATS = 12


def inputs(k, dtype, N, C):
    b = wl.custom(dtype, N, C, seed=9100 + k, dout_sigma=0.02)
    return {name: to_device(getattr(b, name), dtype)
            for name in ("inp", "dout", "weight", "bias")}, b.eps


def run_calls(x, dtype, N, C, eps, stream):
    """Forward, backward and the recomputing accumulating backward, REPEATS
    times, on `stream`; returns the outputs of the last round."""
    tdt = TORCH_DT[dtype]
    code = DT[dtype]
    with torch.cuda.stream(stream):
        out = torch.empty(N, C, dtype=tdt, device="cuda")
        mean = torch.empty(N, device="cuda")
        rstd = torch.empty(N, device="cuda")
        dinp = torch.empty(N, C, dtype=tdt, device="cuda")
        dw = torch.empty(C, device="cuda")
        db = torch.empty(C, device="cuda")
        acc = torch.zeros(N, C, dtype=tdt, device="cuda")
        adw = torch.zeros(C, device="cuda")
        adb = torch.zeros(C, device="cuda")
    for _ in range(REPEATS):
        ln.ln_forward(out, mean, rstd, x["inp"], x["weight"], x["bias"], N, C, eps, code,
                      stream)
        ln.ln_backward(dinp, dw, db, x["dout"], x["inp"], x["weight"], mean, rstd, N, C,
                       code, stream)
        with torch.cuda.stream(stream):
            acc.zero_()
            adw.zero_()
            adb.zero_()
        ln.ln_backward_ex(acc, adw, adb, x["dout"], x["inp"], x["weight"], None, None, N, C,
                          eps, code, ln.LN_BWD_ACCUMULATE_DINP | ln.LN_BWD_ACCUMULATE_DPARAMS
                          | ln.LN_BWD_RECOMPUTE_STATS, stream)
    stream.synchronize()
    return [out, mean, rstd, dinp, dw, db, acc, adw, adb]


def main():
    torch.cuda.init()
    data = [inputs(k, *s) for k, s in enumerate(SHAPES)]
    torch.cuda.synchronize()
    launches0 = ln.launch_count()
    results = [None] * len(SHAPES)
    errors = []
    barrier = threading.Barrier(len(SHAPES))

    def worker(k):
        try:
            dtype, N, C = SHAPES[k]
            x, eps = data[k]
            stream = torch.cuda.Stream()
            barrier.wait()
            results[k] = run_calls(x, dtype, N, C, eps, stream)
        except Exception as e:      # reported below; the test fails on any
            errors.append(f"{SHAPES[k]}: {e!r}")

    threads = [threading.Thread(target=worker, args=(k,)) for k in range(len(SHAPES))]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    threaded_launches = ln.launch_count() - launches0

    mismatches = []
    if not errors:
        serial = torch.cuda.Stream()
        for k, (dtype, N, C) in enumerate(SHAPES):
            x, eps = data[k]
            again = run_calls(x, dtype, N, C, eps, serial)
            for i, (a, b) in enumerate(zip(results[k], again)):
                if not torch.equal(bits(a), bits(b)):
                    mismatches.append(f"{SHAPES[k]} output {i}")
    print(json.dumps({"errors": errors, "mismatches": mismatches,
                      "threaded_launches": threaded_launches,
                      "device_status": ln.device_status()}))


if __name__ == "__main__":
    main()
