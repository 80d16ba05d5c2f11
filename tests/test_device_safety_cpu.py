"""Device code never waits without a bound and never traps (host only).

Every kernel wait in the library is an mbarrier wait, and every such wait
must give up after a bounded number of polls and a bounded time, record the
failure in the device status word and return, so that a stuck copy or a
missing arrival ends the kernel with an error instead of hanging the GPU.  No
kernel may stop the device on purpose either.  These tests read the kernel
sources with comments removed and hold them to that:
  - the mbarrier wait instructions appear only inside the one polling
    helper, and that helper is called only from the bounded wait loop;
  - that loop keeps both its iteration limit and its time limit;
  - no device source has a while loop, an endless for loop, a trap or an
    assert."""
import os
import re

import pytest

import bench

CSRC = os.path.join(bench.ROOT, "layernorm_fwd_bwd_b200", "csrc")
SOURCES = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


def code(path):
    return bench.strip_comments(open(path).read())


@pytest.fixture(scope="module")
def sources():
    return {os.path.basename(p): code(p) for p in SOURCES}


def function_body(text, name):
    """The braces-balanced body of the first definition of `name`."""
    m = re.search(r"\b" + re.escape(name) + r"\s*\([^;{]*\)\s*\{", text)
    assert m, name
    depth, i = 0, m.end() - 1
    for j in range(i, len(text)):
        depth += {"{": 1, "}": -1}.get(text[j], 0)
        if depth == 0:
            return text[i:j + 1]
    raise AssertionError(f"{name}: unbalanced braces")


def test_wait_instructions_only_in_the_polling_helper(sources):
    waits = {f: len(re.findall(r"mbarrier\.(?:try_wait|test_wait)", t)) for f, t in sources.items()}
    assert waits.pop("ln_tma.cuh") == 1, "one mbarrier wait instruction, in mbar_try_wait"
    assert not any(waits.values()), waits
    poll = function_body(sources["ln_tma.cuh"], "mbar_try_wait")
    assert "mbarrier.try_wait" in poll


def test_polling_helper_called_only_from_the_bounded_wait(sources):
    calls = {f: len(re.findall(r"\bmbar_try_wait\s*\(", t)) for f, t in sources.items()}
    tma = sources["ln_tma.cuh"]
    wait = function_body(tma, "mbar_wait")
    in_wait = len(re.findall(r"\bmbar_try_wait\s*\(", wait))
    assert in_wait >= 1
    # the definition itself, plus the calls inside mbar_wait: nothing else
    assert calls.pop("ln_tma.cuh") == 1 + in_wait
    assert not any(calls.values()), calls


def test_the_wait_loop_has_both_limits(sources):
    tma = sources["ln_tma.cuh"]
    wait = function_body(tma, "mbar_wait")
    assert re.search(r"for\s*\([^;]*;\s*it\s*<\s*kMaxWaitIters\s*;", wait), "iteration bound"
    assert "kWaitLimitNs" in wait and "global_ns()" in wait, "time bound"
    assert "return false" in wait, "gives up with a failure"
    limit = re.search(r"kWaitLimitNs\s*=\s*(\d+)ull", tma)
    assert limit and int(limit.group(1)) <= 2_000_000_000, "at most 2 s"
    iters = re.search(r"kMaxWaitIters\s*=\s*([0-9u]+)", tma)
    assert iters, "an iteration cap"


def test_every_bounded_wait_result_is_used(sources):
    """A wait whose result is ignored would carry on over data that never
    arrived: every call of mbar_wait / tile_wait is tested or assigned."""
    for f, t in sources.items():
        for m in re.finditer(r"\b(mbar_wait|tile_wait)\s*\(", t):
            before = t[max(0, m.start() - 40):m.start()]
            if re.search(r"(bool|uint64_t|__forceinline__\s+\w+)\s*$", before):
                continue                        # the definition
            assert re.search(r"(!|=|return|if\s*\(|&&|\|\|)\s*$", before), \
                f"{f}: result of {m.group(1)} unused: ...{before}{m.group(0)}"


@pytest.mark.parametrize("name", [os.path.basename(p) for p in SOURCES])
def test_no_unbounded_loop_or_trap(sources, name):
    t = sources[name]
    assert not re.search(r"\bwhile\s*\(", t), f"{name}: while loop"
    assert not re.search(r"for\s*\(\s*;\s*;\s*\)", t), f"{name}: endless for loop"
    assert not re.search(r"\btrap\b|__trap|\bassert\s*\(|__brkpt", t), f"{name}: trap or assert"
