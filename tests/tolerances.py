"""Parity tolerances between the CUDA library and the CPU oracle.

fp32 tensors: max|gpu - ref| / max|ref| per tensor, at most 1e-5 for out,
mean and rstd and at most 1e-4 for dinp, dweight and dbias.

bf16 tensors (out, dinp): at most 2 bf16 ulps, where the ulp of a reference
value v is 2^(floor(log2 m) - 7) taken at m = max(|v|, 2^-8 * max|ref|).  The
floor keeps elements where the result is near zero (cancellation of fp32
terms of ordinary size) from being judged in ulps of a tiny number; bf16 has
8 significant bits, hence the 7.  mean, rstd, dweight and dbias stay fp32
under bf16 activations: 1e-5 for mean/rstd, 1e-3 for dweight/dbias.

fp16 tensors (no stated tolerance; the same rule carried over to fp16's 11
significant bits): at most 2 fp16 ulps, 2^(floor(log2 m) - 10) at
m = max(|v|, 2^-11 * max|ref|, 2^-14) (2^-14 is fp16's smallest normal, below
which its spacing stays 2^-24); mean/rstd 1e-5, dweight/dbias 1e-3.

These per-tensor rules are the stated ones for the five benchmark workloads.
For other shapes (the sweep: single rows, C = 2, ...) a tensor's max-abs can
be far below the size of the terms it is computed from: the mean of one
N(0, 1) row is ~1/sqrt(C) while its summands are ~1, and for C = 2 dinp is
~eps while rstd * (g - mean(g) - xhat * mean(g xhat)) cancels terms of size
rstd * |g|.  fp32 arithmetic errs in proportion to those terms, so there the
error is measured against ``magnitude_scales``: max|x| for mean,
max_r rstd_r * max_c |dout w| for dinp and max_c sum_r |dout xhat| (resp.
|dout|) for dweight (resp. dbias); the larger of that and max|ref| is the
denominator.
"""
from __future__ import annotations

import numpy as np

FP32_FWD = 1e-5
FP32_BWD = 1e-4
BF16_ULPS = 2.0
BF16_STATS = 1e-5
BF16_PARAM_GRADS = 1e-3


def rel_max(got, ref, scale: float = 0.0) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    scale = max(float(np.max(np.abs(ref))), scale)
    err = float(np.max(np.abs(got - ref)))
    if scale == 0.0:
        return err
    return err / scale


# significant bits and smallest normal of the 16-bit formats
_FMT = {"bf16": (8, 2.0 ** -126), "f16": (11, 2.0 ** -14)}


def ulp_error(got, ref, scale: float = 0.0, dtype: str = "bf16") -> np.ndarray:
    p, min_normal = _FMT[dtype]
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    floor = 2.0 ** -p * max(float(np.max(np.abs(ref))) if ref.size else 0.0, scale)
    m = np.maximum(np.maximum(np.abs(ref), floor), min_normal)
    ulp = np.exp2(np.floor(np.log2(m)) - (p - 1))
    return np.abs(got - ref) / ulp


def bf16_ulp_error(got, ref, scale: float = 0.0) -> np.ndarray:
    return ulp_error(got, ref, scale, "bf16")


def max_ulps(got, ref, scale: float = 0.0, dtype: str = "bf16") -> float:
    e = ulp_error(got, ref, scale, dtype)
    return float(e.max()) if e.size else 0.0


def magnitude_scales(x, dout, w, mean, rstd) -> dict:
    """Size of the terms each result is computed from (float64 inputs)."""
    x, dout = np.asarray(x, np.float64), np.asarray(dout, np.float64)
    w = np.asarray(w, np.float64)
    mean, rstd = np.asarray(mean, np.float64), np.asarray(rstd, np.float64)
    if x.size == 0:
        return {}
    xhat = (x - mean[:, None]) * rstd[:, None]
    return {"mean": float(np.max(np.abs(x))),
            "dinp": float(np.max(rstd * np.max(np.abs(dout * w), axis=1))),
            "dweight": float(np.max(np.sum(np.abs(dout * xhat), axis=0))),
            "dbias": float(np.max(np.sum(np.abs(dout), axis=0)))}


def check(name: str, got, ref, dtype: str, kind: str, scale: float = 0.0) -> dict:
    """kind: 'act_fwd' (out), 'act_bwd' (dinp), 'stats' (mean, rstd),
    'param_grad' (dweight, dbias).  ``scale``: magnitude of the terms the
    result is computed from (0: the tensor's own max-abs alone).  Raises
    AssertionError past tolerance; returns the measured error."""
    if kind in ("act_fwd", "act_bwd") and dtype in ("bf16", "f16"):
        e = max_ulps(got, ref, scale, dtype)
        assert e <= BF16_ULPS, f"{name}: {e:.3f} {dtype} ulps > {BF16_ULPS}"
        return {"name": name, "ulps": e}
    if dtype == "f32":
        tol = FP32_FWD if kind in ("act_fwd", "stats") else FP32_BWD
    else:
        tol = BF16_STATS if kind == "stats" else BF16_PARAM_GRADS
    e = rel_max(got, ref, scale)
    assert e <= tol, f"{name}: relative error {e:.3e} > {tol:.0e}"
    return {"name": name, "rel": e}
