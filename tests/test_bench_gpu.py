"""bench.py on a B200: one short run of each arm in a fresh process, and the
JSON line it prints carries every key the benchmark contract names, with
values of the right kind (the numbers themselves are the benchmark's, not
checked here)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=600)
    assert proc.returncode == 0, proc.stderr[-3000:]
    lines = [l for l in proc.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, proc.stdout[-2000:]
    return json.loads(lines[0])


def check_common(line):
    for key, kind in (("metric", str), ("value", (int, float)), ("unit", str),
                      ("n_gpus", int), ("steps", int), ("warmup", int),
                      ("ms_per_step", (int, float)), ("higher_is_better", bool),
                      ("scaling", str), ("dtype", str), ("data", str), ("config", dict),
                      ("cpu_baseline", dict), ("e2e", dict)):
        assert isinstance(line.get(key), kind), (key, line.get(key))
    assert "vs_baseline" in line and line["vs_baseline"] is None
    assert line["value"] > 0 and line["n_gpus"] == 1 and line["higher_is_better"] is True
    assert "workload" in line["config"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0 and cb["sample"]
    assert cb["host_cores"] == os.cpu_count()
    e2e = line["e2e"]
    for key in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert key in e2e, key


def test_bench_line_contract():
    line = run_bench("--steps", "3", "--warmup", "3", "--no-variants", "--no-workloads",
                     "--e2e-steps", "2", "--cpu-seconds", "0.2")
    check_common(line)
    assert line["steps"] == 3 and line["warmup"] == 3 and line["dtype"] == "f32"
    roof = line["roofline"]
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert roof["achieved"] > 0 and roof["peak"] > 0
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-3
    assert roof["traffic"] is None or roof["traffic"] > 0
    assert line["gpu_launches"] == 3 * 3            # forward, row pass, finalise per step
    assert line["e2e"]["h2d_bytes_per_step"] > 0 and line["e2e"]["d2h_bytes_per_step"] > 0
    clocks = line["clocks"]
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(clocks)


def test_reference_arm_contract():
    line = run_bench("--impl", "reference", "--workload", "fp32_256x768", "--steps", "2",
                     "--warmup", "1")
    check_common(line)
    assert line["impl"] == "reference" and line["dtype"] == "f64"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["e2e"]["value"] == line["value"] == line["cpu_baseline"]["value"]
