"""Kernel selection and launch geometry, checked on the host (no GPU).

``tests/host_geometry.cu`` is compiled with nvcc against the library's own
selection headers.  It visits every vectorised row width (1..2100 16-byte
vectors) for every element type and variant exactly as the launchers do, and
checks coverage, minimality, the range of each kernel family, shared memory
against the per-block limit, ring depth, and the rows-per-block choice of
the forward tiles against a brute-force search.  Here the run must report no
failure, and the choices behind the measured workloads are pinned: they name
the kernels the ncu summaries describe."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "host_geometry.cu")


@pytest.fixture(scope="module")
def run():
    from layernorm_fwd_bwd_b200 import build
    exe = os.path.join(build.BUILD_DIR, "host_geometry")
    deps = [SRC, *build.DEPENDS]
    if not os.path.exists(exe) or any(os.path.getmtime(d) > os.path.getmtime(exe)
                                      for d in deps):
        os.makedirs(build.BUILD_DIR, exist_ok=True)
        subprocess.run([build.nvcc(), *build.ARCH, "-std=c++17", "-o", exe, SRC], check=True,
                       capture_output=True, text=True)
    return subprocess.run([exe], capture_output=True, text=True)


@pytest.fixture(scope="module")
def table(run):
    """{(direction, dtype, mode): [(first nvec, last nvec, variant)]}"""
    out = {}
    for line in run.stdout.splitlines():
        if line.startswith("sel "):
            _, d, t, m, lo, hi, variant = line.split(" ", 6)
            out.setdefault((d, t, int(m)), []).append((int(lo), int(hi), variant))
    return out


def choice(table, direction, dtype, mode, nvec):
    for lo, hi, variant in table[(direction, dtype, mode)]:
        if lo <= nvec <= hi:
            return variant
    raise KeyError(nvec)


def test_no_check_fails(run):
    fails = [l for l in run.stdout.splitlines() if l.startswith("FAIL")]
    assert run.returncode == 0 and not fails, "\n".join(fails[:20]) + run.stderr
    last = run.stdout.splitlines()[-1].split()
    assert last[0] == "checks" and int(last[1]) > 100000 and last[3] == "0"


def test_every_width_is_served(table):
    """Each (direction, dtype, mode) table covers 1..2100 without a gap, and
    only widths past 2048 vectors go to the scalar kernels."""
    assert len(table) == 3 * 2 + 3 * 4
    for key, runs in table.items():
        assert runs[0][0] == 1 and runs[-1][1] == 2100, key
        for (_, hi, _), (lo, _, _) in zip(runs, runs[1:]):
            assert lo == hi + 1, key
        assert [v for lo, hi, v in runs if v == "scalar"] == ["scalar"], key
        assert runs[-1] == (2049, 2100, "scalar"), key


# (direction, dtype, mode, 16-byte vectors per row, variant): mode 1 is the
# residual forward / accumulating backward, 2 the recomputing backward
PINNED = [
    ("fwd", "bf16", 0, 96, "tile V=3 W=1"),              # GPT-2 124M, C = 768
    ("fwd", "bf16", 0, 128, "tile V=4 W=1"),             # GPT-2 350M, C = 1024
    ("fwd", "bf16", 0, 200, "tile V=7 W=1"),             # GPT-2 1.5B, C = 1600
    ("fwd", "f32", 0, 192, "tile V=6 W=1"),              # fp32, C = 768
    ("fwd", "bf16", 1, 96, "tile V=3 W=1"),              # residual forward, C = 768
    ("fwd", "bf16", 0, 384, "tile2 V=6 W=2"),            # C = 3072: two warps per row
    ("fwd", "bf16", 0, 512, "tile2 V=8 W=2"),            # C = 4096
    ("fwd", "bf16", 1, 512, "tile2 V=8 W=2 tiles=1"),    # residual C = 4096: one tile
    ("fwd", "bf16", 0, 1024, "tile4 V=8 W=4 tiles=3"),   # C = 8192: four warps per row
    ("fwd", "bf16", 1, 1024, "tile4 V=8 W=4 tiles=1"),   # residual C = 8192: two arrays
    ("fwd", "bf16", 0, 1025, "vec V=4 W=16"),            # past the four-warp tile
    ("fwd", "bf16", 0, 2000, "vec V=4 W=16"),            # C = 16000
    ("bwd", "bf16", 0, 96, "ring V=3 W=1 S=4"),          # GPT-2 124M
    ("bwd", "bf16", 0, 128, "ring V=4 W=1 S=3"),         # GPT-2 350M
    ("bwd", "bf16", 0, 200, "split VR=7 VC=1 S=4"),      # GPT-2 1.5B: 8 row, 7 column warps
    ("bwd", "bf16", 1, 200, "split VR=7 VC=1 S=2"),      # accumulating 1.5B: three arrays
    ("bwd", "bf16", 2, 200, "ring V=3 W=3 S=4"),         # recomputing 1.5B: three warps per row
    ("bwd", "f32", 0, 192, "ring V=6 W=1 S=2"),          # fp32, C = 768
    ("bwd", "bf16", 1, 96, "ring V=3 W=1 S=3"),          # accumulating: three arrays a stage
    ("bwd", "bf16", 2, 96, "ring V=3 W=1 S=4"),          # recomputing
    ("bwd", "bf16", 2, 128, "ring V=3 W=2 S=4"),         # recomputing C = 1024: two warps
    ("bwd", "f16", 0, 96, "ring V=3 W=1 S=4"),           # fp16 GPT-2 124M shape
    ("bwd", "bf16", 0, 512, "ring V=3 W=6 S=5"),         # C = 4096: six warps per row
    ("bwd", "bf16", 0, 672, "ring V=3 W=7 S=4"),         # C = 5376: the ring's widest row
    ("bwd", "bf16", 0, 673, "vec V=4 W=8"),              # past the ring
]


@pytest.mark.parametrize("direction,dtype,mode,nvec,variant", PINNED)
def test_workload_choices(table, direction, dtype, mode, nvec, variant):
    assert choice(table, direction, dtype, mode, nvec) == variant
