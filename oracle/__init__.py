"""CPU oracle for LayerNorm forward and analytical backward (double precision).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the CUDA library and its Python binding) never imports it, and this package
imports nothing from the product.

The arithmetic lives in ``ln_oracle.c`` (plain loops over the textbook
definition, see that file's header).  This module compiles it with the host C
compiler when the shared object is missing or older than the source, and
exposes it through ctypes on float64 numpy arrays.

Every function is pinned by CPU tests to values fixed by mathematics alone:
closed forms for C = 1 and C = 2, exact power-of-two scaling, constant rows,
finite differences, hand-worked examples under ``tests/golden/`` and
``torch.nn.functional.layer_norm`` in float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "ln_oracle.c")
LIBRARY = os.path.join(_HERE, "libln_oracle.so")

_DBL = ctypes.POINTER(ctypes.c_double)


def compile_oracle(source: str = SOURCE, library: str = LIBRARY) -> str:
    """Compile ``source`` into the shared object ``library`` with gcc (-O2, no
    fast-math, so that every double operation rounds as IEEE 754 says)."""
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", "-o", library, source, "-lm"]
    subprocess.run(cmd, check=True)
    return library


def _stale(source: str, library: str) -> bool:
    return (not os.path.exists(library)
            or os.path.getmtime(library) < os.path.getmtime(source))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_DBL)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


class Oracle:
    """ctypes view of one compiled oracle library (the default one, or a
    deliberately broken copy that a test builds to check that the pins fail)."""

    def __init__(self, library: str = LIBRARY, source: str = SOURCE):
        if library == LIBRARY and _stale(source, library):
            compile_oracle(source, library)
        self.library = library
        lib = ctypes.CDLL(library)
        lib.oracle_ln_forward.restype = ctypes.c_int
        lib.oracle_ln_forward.argtypes = [_DBL, _DBL, _DBL, _DBL, _DBL, _DBL,
                                          ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_double]
        lib.oracle_ln_backward.restype = ctypes.c_int
        lib.oracle_ln_backward.argtypes = [_DBL, _DBL, _DBL, _DBL, _DBL, _DBL,
                                           _DBL, _DBL, ctypes.c_int64,
                                           ctypes.c_int64]
        self._lib = lib

    def forward(self, inp, weight, bias, eps: float):
        """LayerNorm forward of an [N, C] array.  Returns (out [N, C],
        mean [N], rstd [N]) in float64."""
        x = _f64(inp)
        if x.ndim != 2:
            raise ValueError("inp must be 2-D [N, C]")
        n, c = x.shape
        w, b = _f64(weight).reshape(-1), _f64(bias).reshape(-1)
        if w.size != c or b.size != c:
            raise ValueError("weight and bias must hold C values")
        out = np.empty((n, c), np.float64)
        mean = np.empty(n, np.float64)
        rstd = np.empty(n, np.float64)
        rc = self._lib.oracle_ln_forward(_ptr(out), _ptr(mean), _ptr(rstd),
                                         _ptr(x), _ptr(w), _ptr(b), n, c,
                                         float(eps))
        if rc != 0:
            raise ValueError(f"oracle_ln_forward rejected N={n} C={c} ({rc})")
        return out, mean, rstd

    def backward(self, dout, inp, weight, mean, rstd):
        """Analytical backward given the saved per-row statistics.  Returns
        (dinp [N, C], dweight [C], dbias [C]) in float64."""
        x = _f64(inp)
        dy = _f64(dout)
        if x.ndim != 2 or dy.shape != x.shape:
            raise ValueError("inp and dout must be 2-D arrays of one shape")
        n, c = x.shape
        w = _f64(weight).reshape(-1)
        m, s = _f64(mean).reshape(-1), _f64(rstd).reshape(-1)
        if w.size != c or m.size != n or s.size != n:
            raise ValueError("weight must hold C values, mean/rstd N values")
        dinp = np.empty((n, c), np.float64)
        dweight = np.empty(c, np.float64)
        dbias = np.empty(c, np.float64)
        rc = self._lib.oracle_ln_backward(_ptr(dinp), _ptr(dweight),
                                          _ptr(dbias), _ptr(dy), _ptr(x),
                                          _ptr(w), _ptr(m), _ptr(s), n, c)
        if rc != 0:
            raise ValueError(f"oracle_ln_backward rejected N={n} C={c} ({rc})")
        return dinp, dweight, dbias


_default: Oracle | None = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def ln_forward(inp, weight, bias, eps: float):
    return default().forward(inp, weight, bias, eps)


def ln_backward(dout, inp, weight, mean, rstd):
    return default().backward(dout, inp, weight, mean, rstd)
