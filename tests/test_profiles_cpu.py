"""The committed ncu summaries (host only): short text that gives the full
command that made it, runs committed files only, leaves the GPU clocks alone,
and still parses against the benchmark it names."""
import os
import re
import shlex
import subprocess
import sys

import pytest

import bench

PROFILES = os.path.join(bench.ROOT, "profiles")
FILES = sorted(f for f in os.listdir(PROFILES))


def commands(text):
    """Indented command lines with their backslash continuations joined."""
    lines, out, cur = text.splitlines(), [], ""
    for line in lines:
        if not line.startswith("    ") and not cur:
            continue
        cur += " " + line.strip().rstrip("\\").strip()
        if not line.rstrip().endswith("\\"):
            out.append(cur.strip())
            cur = ""
    return [c for c in out if c.startswith(("python ", "ncu ")) or " ncu " in c]


def test_profiles_are_short_text():
    tracked = subprocess.run(["git", "ls-files", "profiles"], cwd=bench.ROOT, capture_output=True,
                             text=True, check=True).stdout.split()
    assert tracked, "profiles/ holds the ncu summaries"
    for f in FILES:
        assert f.endswith((".md", ".txt")), f"{f}: summaries only, no raw reports"
        assert os.path.getsize(os.path.join(PROFILES, f)) < 16 * 1024, f"{f}: keep it short"


@pytest.mark.parametrize("name", FILES)
def test_every_capture_states_its_command(name):
    text = open(os.path.join(PROFILES, name)).read()
    cmds = commands(text)
    referenced = re.findall(r"same capture as (\S+\.md)", text)
    assert cmds or referenced, f"{name}: no command and no reference to the capture it shares"
    for other in referenced:
        assert other in FILES, f"{name}: refers to missing {other}"
    assert "_work" not in text, f"{name}: commands must run committed files only"


@pytest.mark.parametrize("name", FILES)
def test_ncu_leaves_the_clocks_alone(name):
    for c in commands(open(os.path.join(PROFILES, name)).read()):
        for part in re.split(r";|&&|\bdo\b", c):
            part = part.strip()
            if part.startswith("ncu ") and " -i " not in f" {part} ":
                assert "--clock-control none" in part, f"{name}: {part}"


@pytest.mark.parametrize("name", FILES)
def test_bench_commands_still_parse(name, monkeypatch):
    """Every `python bench.py ...` in a summary is accepted by today's
    bench.py argument parser, with a workload it knows."""
    from layernorm_fwd_bwd_b200 import workloads as wl
    for c in commands(open(os.path.join(PROFILES, name)).read()):
        for m in re.finditer(r"python bench\.py((?:\s+--?[\w-]+(?:\s+[\w.]+)?)*)", c):
            argv = shlex.split(m.group(1))
            monkeypatch.setattr(sys, "argv", ["bench.py", *argv])
            args = bench.parse_args()
            assert args.workload in wl.WORKLOADS, f"{name}: {args.workload}"


def test_traffic_profile_is_machine_readable():
    text = open(bench.TRAFFIC_PROFILE).read()
    assert re.search(r"dram_bytes_per_call:\s*\d+", text)
    assert re.search(r"kernel_source_sha256:\s*[0-9a-f]{64}", text)
