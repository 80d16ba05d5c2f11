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
``torch.nn.functional.layer_norm`` in float64; the rounding routine by brute
force over every value of each format and by numpy's casts; the backward
variants by the linearity of the gradient in dout and by torch's autograd,
which recomputes the statistics itself.
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

# Binary floating-point formats as (significant bits p, minimum normal
# exponent emin, largest finite value), IEEE 754 parameters.
FORMATS = {
    "f32": (24, -126, (2.0 - 2.0 ** -23) * 2.0 ** 127),
    "bf16": (8, -126, (2.0 - 2.0 ** -7) * 2.0 ** 127),
    "f16": (11, -14, 65504.0),
}


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
        lib.oracle_round_format.restype = ctypes.c_int
        lib.oracle_round_format.argtypes = [_DBL, _DBL, ctypes.c_int64, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_double]
        lib.oracle_ln_forward_residual.restype = ctypes.c_int
        lib.oracle_ln_forward_residual.argtypes = [
            _DBL, _DBL, _DBL, _DBL, _DBL, _DBL, _DBL, _DBL, ctypes.c_int64,
            ctypes.c_int64, ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_double]
        lib.oracle_ln_backward_ex.restype = ctypes.c_int
        lib.oracle_ln_backward_ex.argtypes = [
            _DBL, _DBL, _DBL, _DBL, _DBL, _DBL, _DBL, _DBL, ctypes.c_int64,
            ctypes.c_int64, ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int]
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


    def round_to(self, values, fmt: str) -> np.ndarray:
        """Each value rounded to the nearest value of ``fmt`` ("f32", "bf16",
        "f16"), ties to even, overflow to infinity."""
        v = _f64(values)
        out = np.empty_like(v)
        p, emin, top = FORMATS[fmt]
        rc = self._lib.oracle_round_format(_ptr(out), _ptr(v), v.size, p, emin, top)
        if rc != 0:
            raise ValueError(f"oracle_round_format rejected {fmt} ({rc})")
        return out

    def forward_residual(self, resid, branch, weight, bias, eps: float, fmt: str):
        """Forward of x = round_fmt(resid + branch).  Returns (x, out, mean,
        rstd) in float64."""
        a, b = _f64(resid), _f64(branch)
        if a.ndim != 2 or b.shape != a.shape:
            raise ValueError("resid and branch must be 2-D arrays of one shape")
        n, c = a.shape
        w, bb = _f64(weight).reshape(-1), _f64(bias).reshape(-1)
        if w.size != c or bb.size != c:
            raise ValueError("weight and bias must hold C values")
        x = np.empty((n, c), np.float64)
        out = np.empty((n, c), np.float64)
        mean = np.empty(n, np.float64)
        rstd = np.empty(n, np.float64)
        p, emin, top = FORMATS[fmt]
        rc = self._lib.oracle_ln_forward_residual(
            _ptr(x), _ptr(out), _ptr(mean), _ptr(rstd), _ptr(a), _ptr(b), _ptr(w),
            _ptr(bb), n, c, float(eps), p, emin, top)
        if rc != 0:
            raise ValueError(f"oracle_ln_forward_residual rejected N={n} C={c} ({rc})")
        return x, out, mean, rstd

    def backward_ex(self, dout, inp, weight, mean=None, rstd=None, eps: float = 0.0,
                    dinp_prev=None, dweight_prev=None, dbias_prev=None,
                    recompute: bool = False):
        """Backward variants: with ``recompute`` mean/rstd are recomputed from
        inp with eps (the arguments are ignored); a ``*_prev`` array given
        means that gradient is added to it (dinp_prev, or both dweight_prev
        and dbias_prev).  Returns (dinp, dweight, dbias) in float64."""
        x = _f64(inp)
        dy = _f64(dout)
        if x.ndim != 2 or dy.shape != x.shape:
            raise ValueError("inp and dout must be 2-D arrays of one shape")
        n, c = x.shape
        w = _f64(weight).reshape(-1)
        if (dweight_prev is None) != (dbias_prev is None):
            raise ValueError("give both dweight_prev and dbias_prev, or neither")
        m = np.zeros(n) if recompute else _f64(mean).reshape(-1)
        s = np.zeros(n) if recompute else _f64(rstd).reshape(-1)
        if w.size != c or m.size != n or s.size != n:
            raise ValueError("weight must hold C values, mean/rstd N values")
        dinp = (np.zeros((n, c)) if dinp_prev is None
                else np.array(_f64(dinp_prev).reshape(n, c), copy=True))
        dweight = np.zeros(c) if dweight_prev is None else np.array(_f64(dweight_prev), copy=True)
        dbias = np.zeros(c) if dbias_prev is None else np.array(_f64(dbias_prev), copy=True)
        rc = self._lib.oracle_ln_backward_ex(
            _ptr(dinp), _ptr(dweight), _ptr(dbias), _ptr(dy), _ptr(x), _ptr(w), _ptr(m),
            _ptr(s), n, c, float(eps), int(dinp_prev is not None),
            int(dweight_prev is not None), int(bool(recompute)))
        if rc != 0:
            raise ValueError(f"oracle_ln_backward_ex rejected N={n} C={c} ({rc})")
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
