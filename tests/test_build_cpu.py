"""The build's resource report (host only): ptxas prints, for every kernel of
every object, its registers, stack frame and spill bytes (``-Xptxas=-v``;
the build keeps the report beside each object).  The kernels the measured
workloads run must not spill; every other kernel stays within a small,
stated bound.  A change that makes a hot kernel spill, or any kernel spill
heavily, fails here before it reaches a GPU."""
import os
import re

import pytest

ENTRY = re.compile(r"Compiling entry function '(\S+)' for 'sm_100a'\n"
                   r".*\n\s*(\d+) bytes stack frame, (\d+) bytes spill stores, "
                   r"(\d+) bytes spill loads\n.*Used (\d+) registers")

# Kernels of the measured workloads (mangled-name prefixes; template arguments
# T, V, warps, stages or tiles, ..., W, MODE): no spill at all.
NO_SPILL = {
    "forward bf16 C=768 (one warp, 3 vectors, full rows)":
        "_ZN3lnk18ln_fwd_tile_kernelI13__nv_bfloat16Li3ELi8ELi2ELi1ELb1ELi0E",
    "forward bf16 C=1024": "_ZN3lnk18ln_fwd_tile_kernelI13__nv_bfloat16Li4ELi8ELi2ELi1ELb1ELi0E",
    "residual forward bf16 C=768":
        "_ZN3lnk18ln_fwd_tile_kernelI13__nv_bfloat16Li3ELi8ELi2ELi1ELb1ELi1E",
    "forward fp16 C=768": "_ZN3lnk18ln_fwd_tile_kernelI6__halfLi3ELi8ELi2ELi1ELb1ELi0E",
    "backward bf16 C=768 (ring, 4 stages)":
        "_ZN3lnk17ln_bwd_tma_kernelI13__nv_bfloat16Li3ELi15ELi4ELb1ELi1ELi0E",
    "backward bf16 C=1024 (ring, 4 vectors)":
        "_ZN3lnk17ln_bwd_tma_kernelI13__nv_bfloat16Li4ELi15ELi3ELb1ELi1ELi0E",
    "accumulating backward bf16 C=768 (3 stages)":
        "_ZN3lnk17ln_bwd_tma_kernelI13__nv_bfloat16Li3ELi15ELi3ELb1ELi1ELi1E",
    "recomputing backward bf16 C=768":
        "_ZN3lnk17ln_bwd_tma_kernelI13__nv_bfloat16Li3ELi15ELi4ELb1ELi1ELi2E",
    "backward fp16 C=768": "_ZN3lnk17ln_bwd_tma_kernelI6__halfLi3ELi15ELi4ELb1ELi1ELi0E",
    "backward fp32 C=768 (ring, 6 vectors)":
        "_ZN3lnk17ln_bwd_tma_kernelIfLi6ELi15ELi2ELb1ELi1ELi0E",
    "backward bf16 C=1600 (split: 8 row warps, 7 column warps)":
        "_ZN3lnk19ln_bwd_split_kernelI13__nv_bfloat16Li7ELi1ELi8ELi7ELi0E",
    "accumulating backward bf16 C=1600 (split)":
        "_ZN3lnk19ln_bwd_split_kernelI13__nv_bfloat16Li7ELi1ELi8ELi7ELi1E",
    "backward bf16 C=2048 (split: 8 row warps, 4 column warps)":
        "_ZN3lnk19ln_bwd_split_kernelI13__nv_bfloat16Li8ELi2ELi8ELi4ELi0E",
    "column finalise": "_ZN3lnk16ln_colsum_kernelEPfS0_PKfiii",
}
# Every kernel: spill stores and loads, and the stack frame, at most this
# many bytes.  Today's largest are the 16-bit one-warp forward tiles of 8
# vectors per lane, held to 80 registers for 3 resident blocks per SM
# (measured faster than more registers and fewer blocks).
MAX_SPILL_BYTES = 128


@pytest.fixture(scope="module")
def kernels():
    from layernorm_fwd_bwd_b200 import build
    build.build()
    if not all(os.path.exists(build.ptxas_report(o)) for o in build.objects()):
        build.build(force=True)      # a library built before reports were kept
    out = {}
    for obj in build.objects():
        text = open(build.ptxas_report(obj)).read()
        for name, stack, st, ld, regs in ENTRY.findall(text):
            out[name] = dict(obj=os.path.basename(obj), stack=int(stack), spill_st=int(st),
                             spill_ld=int(ld), regs=int(regs))
    return out


def test_every_object_reports_its_kernels(kernels):
    from layernorm_fwd_bwd_b200 import build
    objs = {k["obj"] for k in kernels.values()}
    inst = {os.path.basename(o) for o in build.objects() if "ln_inst_" in o}
    assert inst <= objs, sorted(inst - objs)
    assert len(kernels) > 200


@pytest.mark.parametrize("what", sorted(NO_SPILL))
def test_measured_kernels_do_not_spill(kernels, what):
    prefix = NO_SPILL[what]
    hits = [(n, k) for n, k in kernels.items() if n.startswith(prefix)]
    assert len(hits) == 1, f"{what}: {len(hits)} kernels match {prefix}"
    name, k = hits[0]
    assert k["spill_st"] == 0 and k["spill_ld"] == 0 and k["stack"] == 0, (what, k)
    assert k["regs"] <= 128, (what, k)       # 512-thread rings, 1 block per SM


def test_no_kernel_spills_heavily(kernels):
    heavy = {n: k for n, k in kernels.items()
             if max(k["spill_st"], k["spill_ld"], k["stack"]) > MAX_SPILL_BYTES}
    assert not heavy, heavy


def test_no_compiler_warnings(kernels):
    """Every object compiles without a compiler warning (for example #1886-D,
    which nvcc gives when two kernels declare the dynamic shared array with
    different alignments)."""
    from layernorm_fwd_bwd_b200 import build
    for obj in build.objects():
        text = open(build.ptxas_report(obj)).read()
        warnings = [line for line in text.splitlines() if re.search(r"\bwarning\b", line)]
        assert not warnings, f"{os.path.basename(obj)}: {warnings[:3]}"
