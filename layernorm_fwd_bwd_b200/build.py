"""Build libln.so in-tree with nvcc for sm_100a.

    python -m layernorm_fwd_bwd_b200.build [--verbose]

The shared object lands next to this file (``layernorm_fwd_bwd_b200/libln.so``)
and links the CUDA runtime statically, so it does not depend on which
libcudart the host process (for example PyTorch) has loaded.

The kernels are compiled in parallel, one object per (direction, element type,
variant) from ``csrc/ln_inst.cu``, plus the API and no-alloc units; objects go
to ``_build/`` beside this file and are linked into the one library.  ptxas
reports each kernel's registers, stack and spills (``-Xptxas=-v``, which only
prints); the report of each object is kept beside it as ``<object>.ptxas.txt``
(``--verbose`` also prints it).
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(PKG, "_build")
LIBRARY = os.path.join(PKG, "libln.so")

# (direction, element type, variant): direction 0 forward / 1 backward;
# type 0 fp32 / 1 bf16 / 2 fp16; forward variants 0 plain / 1 residual,
# backward variants bit 0 accumulate dinp, bit 1 recompute the statistics.
INSTANCES = [(0, t, m) for t in (0, 1, 2) for m in (0, 1)] + \
            [(1, t, m) for t in (0, 1, 2) for m in (0, 1, 2, 3)]
UNITS = ["ln_api.cu", "ln_noalloc.cu"]
DEPENDS = [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))
           if f.endswith((".cu", ".cuh"))] + [os.path.join(INCLUDE, "ln.h")]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC"]
LINK_FLAGS = ["-shared", "-cudart", "static", *ARCH]


def nvcc() -> str:
    for cand in (os.environ.get("CUDA_HOME", ""), "/usr/local/cuda"):
        path = os.path.join(cand, "bin", "nvcc") if cand else ""
        if path and os.path.exists(path):
            return path
    return "nvcc"


def stale() -> bool:
    if not os.path.exists(LIBRARY):
        return True
    t = os.path.getmtime(LIBRARY)
    return any(os.path.getmtime(p) > t for p in DEPENDS)


def ptxas_report(obj: str) -> str:
    """Path of the ptxas resource report kept for one object."""
    return obj + ".ptxas.txt"


def objects() -> list[str]:
    """Every object the library links."""
    return [obj for obj, _ in _jobs()]


def _jobs() -> list[tuple[str, list[str]]]:
    base = [nvcc(), *NVCC_FLAGS, "-Xptxas=-v", "-I", INCLUDE]
    jobs = []
    for unit in UNITS:
        obj = os.path.join(BUILD_DIR, unit.replace(".cu", ".o"))
        jobs.append((obj, [*base, "-c", os.path.join(CSRC, unit), "-o", obj]))
    for d, t, m in INSTANCES:
        obj = os.path.join(BUILD_DIR, f"ln_inst_{'fb'[d]}{t}{m}.o")
        defs = [f"-DLN_INST_DIR={d}", f"-DLN_INST_T={t}", f"-DLN_INST_MODE={m}"]
        jobs.append((obj, [*base, *defs, "-c", os.path.join(CSRC, "ln_inst.cu"), "-o", obj]))
    return jobs


def build(verbose: bool = False, force: bool = False) -> str:
    if not force and not stale():
        return LIBRARY
    os.makedirs(BUILD_DIR, exist_ok=True)
    jobs = _jobs()

    def compile_one(job):
        return subprocess.run(job[1], capture_output=True, text=True)

    workers = max(1, min(len(jobs), os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=workers) as pool:
        results = list(pool.map(compile_one, jobs))
    failed = False
    for (obj, cmd), res in zip(jobs, results):
        if verbose or res.returncode != 0:
            sys.stderr.write(f"== {os.path.basename(obj)}\n{res.stdout}{res.stderr}")
        failed |= res.returncode != 0
        if res.returncode == 0:
            with open(ptxas_report(obj), "w") as f:
                f.write(res.stdout + res.stderr)
    if failed:
        raise RuntimeError("nvcc failed (see the messages above)")
    link = [nvcc(), *LINK_FLAGS, "-o", LIBRARY + ".tmp", *[obj for obj, _ in jobs]]
    subprocess.run(link, check=True)
    os.replace(LIBRARY + ".tmp", LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force=True))
