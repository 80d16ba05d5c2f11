"""Build libln.so in-tree with nvcc for sm_100a.

    python -m layernorm_fwd_bwd_b200.build [--verbose]

The shared object lands next to this file (``layernorm_fwd_bwd_b200/libln.so``)
and links the CUDA runtime statically, so it does not depend on which
libcudart the host process (for example PyTorch) has loaded.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libln.so")
SOURCES = [os.path.join(CSRC, "ln_api.cu"), os.path.join(CSRC, "ln_noalloc.cu")]
DEPENDS = SOURCES + [os.path.join(CSRC, "ln_kernels.cuh"), os.path.join(CSRC, "ln_select.cuh"),
                     os.path.join(CSRC, "ln_tma.cuh"),
                     os.path.join(CSRC, "ln_tile.cuh"),
                     os.path.join(INCLUDE, "ln.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
]


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


def build(verbose: bool = False, force: bool = False) -> str:
    if not force and not stale():
        return LIBRARY
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-o", LIBRARY + ".tmp", *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(LIBRARY + ".tmp", LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force=True))
