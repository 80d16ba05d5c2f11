"""Pins of the CPU oracle to results fixed by mathematics, not by the oracle.

Each ``pin_*`` function takes an oracle object (``oracle.Oracle``) and raises
AssertionError when the oracle disagrees with the fact it pins.  They run
against the real oracle in ``test_oracle_pins.py`` and against deliberately
broken copies of it in ``test_oracle_mutants.py``, which checks that every
plausible mistake (a dropped term, a wrong sign, a wrong divisor, eps outside
the root, swapped operands) fails at least one pin.

What pins what:
  forward  -- C = 1 closed form, C = 2 closed form, constant rows, exact
              power-of-two scaling (x -> 2x, eps -> 4 eps), shift invariance,
              the moments of the output with unit affine parameters (against
              numpy's biased variance), hand-worked examples, and
              torch.nn.functional.layer_norm in float64;
  backward -- C = 1 and C = 2 closed forms (from differentiating the C = 2
              normalisation by hand), central finite differences of
              L = sum(out * dout) through the forward, the per-row identities
              sum_c dinp = 0 and sum_c dinp * xhat = rstd * eps/(var+eps) *
              sum_c g * xhat, exact integer column sums for dbias, hand-worked
              examples, and torch autograd in float64;
  rounding -- brute force: every finite value of bfloat16 and fp16 (and the
              fp32 values near each probe) enumerated from its bit pattern,
              the nearest chosen with exact rational arithmetic, ties to the
              even bit pattern; numpy's float32 and float16 casts;
  residual forward -- the rounded sum against that brute force on the exact
              (rational) sum, and branch = 0 reducing to the plain forward;
  backward variants -- linearity of the gradient in dout (accumulating the
              gradient of dout1 into that of dout2 gives the gradient of
              dout1 + dout2) and torch autograd in float64, which computes the
              statistics itself (the recomputing variant).
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "hand_worked.txt")


def _rng(seed):
    return np.random.default_rng(seed)


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    scale = max(1e-300, float(np.max(np.abs(b))) if b.size else 1.0)
    return float(np.max(np.abs(a - b))) / scale if a.size else 0.0


# ----------------------------------------------------------------- forward pins

def pin_one_column(orc):
    """C = 1: the row's only deviation is 0, so var = 0, rstd = eps^-1/2,
    out = b exactly, mean = x exactly; every xhat is 0, so dinp = 0 and
    dweight = 0 exactly, and dbias is the plain sum of dout."""
    rng = _rng(1)
    x = rng.normal(size=(7, 1))
    w, b = np.array([1.7]), np.array([-0.3])
    for eps in (1e-5, 0.25, 3.0):
        out, mean, rstd = orc.forward(x, w, b, eps)
        assert np.array_equal(out, np.full_like(out, b[0])), "C=1 out must equal b"
        assert np.array_equal(mean, x[:, 0]), "C=1 mean must equal x"
        assert _rel(rstd, np.full(7, eps ** -0.5)) < 1e-15, "C=1 rstd must be eps^-1/2"
        dout = rng.normal(size=(7, 1))
        dinp, dw, db = orc.backward(dout, x, w, mean, rstd)
        assert np.array_equal(dinp, np.zeros_like(dinp)), "C=1 dinp must be 0"
        assert np.array_equal(dw, np.zeros(1)), "C=1 dweight must be 0"
        assert _rel(db, dout.sum(axis=0)) < 1e-15


def pin_two_columns(orc):
    """C = 2 with x = (a - d, a + d): mean = a, var = d^2, rstd = (d^2+eps)^-1/2,
    xhat = (-d, d) * rstd.  With u = (x1 - x2)/2 = -d, xhat_1 = u/sqrt(u^2+eps)
    and L = (dout1 w1 - dout2 w2) xhat_1 + const, so
    dinp_1 = -dinp_2 = (dout1 w1 - dout2 w2) * eps / (2 (u^2+eps)^(3/2))."""
    rng = _rng(2)
    n = 9
    a = np.round(rng.normal(size=n) * 64) / 64          # dyadic: exact sums
    d = np.round(rng.normal(size=n) * 64) / 64
    x = np.stack([a - d, a + d], axis=1)
    w = np.array([1.25, -0.75])
    b = np.array([0.5, 0.125])
    for eps in (1e-5, 0.5):
        out, mean, rstd = orc.forward(x, w, b, eps)
        q = d * d + eps
        assert _rel(mean, a) < 1e-15
        assert _rel(rstd, 1.0 / np.sqrt(q)) < 1e-14
        xhat = np.stack([-d, d], axis=1) / np.sqrt(q)[:, None]
        assert _rel(out, xhat * w + b) < 1e-14, "C=2 out closed form"
        dout = rng.normal(size=(n, 2))
        dinp, dw, db = orc.backward(dout, x, w, mean, rstd)
        dl_du = (dout[:, 0] * w[0] - dout[:, 1] * w[1]) * eps / q ** 1.5
        want = np.stack([dl_du / 2, -dl_du / 2], axis=1)
        assert _rel(dinp, want) < 1e-12, "C=2 dinp closed form"
        assert _rel(dw, (dout * xhat).sum(axis=0)) < 1e-13
        assert _rel(db, dout.sum(axis=0)) < 1e-15


def pin_constant_rows(orc):
    """A row of one fp32 value v (C <= 768 copies sum exactly in double):
    mean = v exactly, var = 0, out = b exactly, rstd = eps^-1/2, and the
    backward reduces to dinp = rstd * (g - mean(g)) with dweight = 0."""
    rng = _rng(3)
    C = 768
    v = (100.0 + 0.01 * rng.normal(size=5)).astype(np.float32).astype(np.float64)
    x = np.repeat(v[:, None], C, axis=1)
    w = 1.0 + 0.1 * rng.normal(size=C)
    b = 0.1 * rng.normal(size=C)
    eps = float(np.float32(1e-5))
    out, mean, rstd = orc.forward(x, w, b, eps)
    assert np.array_equal(mean, v), "constant row mean must be exact"
    assert np.array_equal(out, np.broadcast_to(b, out.shape)), "constant row out must be b"
    assert _rel(rstd, np.full(5, eps ** -0.5)) < 1e-15
    dout = rng.normal(size=(5, C))
    dinp, dw, db = orc.backward(dout, x, w, mean, rstd)
    g = dout * w
    assert _rel(dinp, rstd[:, None] * (g - g.mean(axis=1, keepdims=True))) < 1e-13
    assert np.array_equal(dw, np.zeros(C))


def pin_scale_by_two(orc):
    """LayerNorm(2x; eps' = 4 eps) = LayerNorm(x; eps) exactly: every sum,
    deviation and square scales by a power of two without rounding, and
    sqrt(4 v) = 2 sqrt(v) exactly.  So mean doubles, rstd halves and out is
    bitwise equal; the backward then gives dinp/2 and identical dweight and
    dbias.  Fails if eps is not inside the root, or not added to the variance."""
    rng = _rng(4)
    x = rng.normal(size=(6, 33))
    w = 1.0 + 0.1 * rng.normal(size=33)
    b = 0.1 * rng.normal(size=33)
    dout = rng.normal(size=(6, 33))
    eps = 0.3
    o1, m1, r1 = orc.forward(x, w, b, eps)
    o2, m2, r2 = orc.forward(2 * x, w, b, 4 * eps)
    assert np.array_equal(m2, 2 * m1)
    assert np.array_equal(r2, r1 / 2)
    assert np.array_equal(o2, o1), "out must be invariant under x->2x, eps->4eps"
    d1, w1, b1 = orc.backward(dout, x, w, m1, r1)
    d2, w2, b2 = orc.backward(dout, 2 * x, w, m2, r2)
    assert np.array_equal(d2, d1 / 2)
    assert np.array_equal(w2, w1) and np.array_equal(b2, b1)


def pin_shift_invariance(orc):
    """Adding a constant k to a row leaves out, rstd and dinp unchanged and
    moves the mean by k."""
    rng = _rng(5)
    x = rng.normal(size=(4, 50))
    w = 1.0 + 0.1 * rng.normal(size=50)
    b = 0.1 * rng.normal(size=50)
    eps = 1e-5
    o1, m1, r1 = orc.forward(x, w, b, eps)
    o2, m2, r2 = orc.forward(x + 37.0, w, b, eps)
    assert _rel(o2, o1) < 1e-12
    assert _rel(m2, m1 + 37.0) < 1e-15
    assert _rel(r2, r1) < 1e-12


def pin_unit_affine_moments(orc):
    """With w = 1 and b = 0 each output row has mean 0 and (biased) variance
    var(x) / (var(x) + eps), var taken by numpy's biased np.var."""
    rng = _rng(6)
    x = rng.normal(size=(8, 97)) * rng.uniform(0.001, 10, size=(8, 1)) + 3.0
    C = x.shape[1]
    for eps in (1e-5, 0.01):
        out, mean, rstd = orc.forward(x, np.ones(C), np.zeros(C), eps)
        assert np.max(np.abs(out.mean(axis=1))) < 1e-12, "output rows must have mean 0"
        v = np.var(x, axis=1)
        assert _rel(np.var(out, axis=1), v / (v + eps)) < 1e-12, "output variance"
        assert _rel(mean, x.mean(axis=1)) < 1e-14
        assert _rel(rstd, 1.0 / np.sqrt(v + eps)) < 1e-12


# ---------------------------------------------------------------- backward pins

def pin_finite_differences(orc):
    """Central differences of L = sum(out * dout) through the oracle's own
    forward agree with its analytical backward on tiny inputs."""
    rng = _rng(7)
    for (n, C, eps) in ((3, 5, 1e-5), (2, 8, 0.1), (4, 2, 0.05), (1, 3, 1.0)):
        x = rng.normal(size=(n, C))
        w = 1.0 + 0.3 * rng.normal(size=C)
        b = 0.3 * rng.normal(size=C)
        dout = rng.normal(size=(n, C))

        def loss(xx, ww, bb):
            return float(np.sum(orc.forward(xx, ww, bb, eps)[0] * dout))

        _, mean, rstd = orc.forward(x, w, b, eps)
        dinp, dw, db = orc.backward(dout, x, w, mean, rstd)

        def fd(arr, which):
            g = np.zeros_like(arr)
            it = np.nditer(arr, flags=["multi_index"])
            for _ in it:
                i = it.multi_index
                h = 1e-6 * max(1.0, abs(arr[i]))
                up, dn = arr.copy(), arr.copy()
                up[i] += h
                dn[i] -= h
                args_up = [x, w, b]
                args_dn = [x, w, b]
                args_up[which], args_dn[which] = up, dn
                g[i] = (loss(*args_up) - loss(*args_dn)) / (up[i] - dn[i])
            return g

        for name, an, which, arr in (("dinp", dinp, 0, x), ("dweight", dw, 1, w),
                                     ("dbias", db, 2, b)):
            num = fd(arr, which)
            err = np.max(np.abs(num - an)) / max(1.0, np.max(np.abs(an)))
            assert err < 1e-6, f"finite differences disagree on {name}: {err:.2e}"


def pin_row_identities(orc):
    """Per row: sum_c dinp = 0, and with xhat and g = dout * w,
    sum_c dinp * xhat = rstd * eps / (var + eps) * sum_c g * xhat
    (because sum_c xhat^2 = C var / (var + eps)); this tends to 0 as eps -> 0."""
    rng = _rng(8)
    x = rng.normal(size=(6, 40)) * 0.05 + 2.0
    w = 1.0 + 0.1 * rng.normal(size=40)
    b = np.zeros(40)
    dout = rng.normal(size=(6, 40))
    eps = 1e-3
    _, mean, rstd = orc.forward(x, w, b, eps)
    dinp, _, _ = orc.backward(dout, x, w, mean, rstd)
    var = np.var(x, axis=1)
    xhat = (x - x.mean(axis=1, keepdims=True)) / np.sqrt(var + eps)[:, None]
    g = dout * w
    scale = np.sum(np.abs(dinp), axis=1)
    assert np.all(np.abs(dinp.sum(axis=1)) <= 1e-13 * scale), "sum dinp must be 0"
    want = (1.0 / np.sqrt(var + eps)) * eps / (var + eps) * np.sum(g * xhat, axis=1)
    got = np.sum(dinp * xhat, axis=1)
    assert np.all(np.abs(got - want) <= 1e-9 * np.sum(np.abs(dinp * xhat), axis=1)), \
        "sum dinp*xhat closed form"


def pin_dbias_integer_sum(orc):
    """dbias is the column sum of dout: exact for small-integer dout; with
    xhat computed from given statistics, dweight = sum_r dout * xhat is exact
    too when xhat is a small dyadic number."""
    rng = _rng(9)
    n, C = 50, 12
    x = rng.integers(-8, 9, size=(n, C)).astype(np.float64)
    dout = rng.integers(-5, 6, size=(n, C)).astype(np.float64)
    w = np.ones(C)
    mean = np.zeros(n)
    rstd = np.full(n, 0.25)
    dinp, dw, db = orc.backward(dout, x, w, mean, rstd)
    assert np.array_equal(db, dout.sum(axis=0)), "dbias must be the column sum"
    assert np.array_equal(dw, (dout * x * 0.25).sum(axis=0)), "dweight column sum"


# ----------------------------------------------------------------- golden files

def load_golden(path: str = GOLDEN):
    cases, cur = [], None
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            if key == "case":
                cur = {"name": val}
                cases.append(cur)
                continue
            rows = [[float(Fraction(t)) for t in r.split()] for r in val.split(";")]
            cur[key] = np.array(rows, np.float64)
    return cases


def pin_hand_worked(orc):
    """Hand-worked examples in tests/golden/hand_worked.txt."""
    for case in load_golden():
        eps = float(case["eps"][0, 0])
        out, mean, rstd = orc.forward(case["x"], case["w"][0], case["b"][0], eps)
        for key, got in (("out", out), ("mean", mean), ("rstd", rstd)):
            assert _rel(got, case[key].reshape(got.shape)) < 1e-14, \
                f"{case['name']}: {key}"
        dinp, dw, db = orc.backward(case["dout"], case["x"], case["w"][0], mean, rstd)
        for key, got in (("dinp", dinp), ("dweight", dw), ("dbias", db)):
            assert np.max(np.abs(got - case[key].reshape(got.shape))) < 1e-14, \
                f"{case['name']}: {key}"


# ------------------------------------------------------------ library cross-check

def pin_torch_float64(orc):
    """torch.nn.functional.layer_norm in float64 on the CPU (a library routine
    computing the same definition) and its autograd gradients."""
    import torch
    rng = _rng(10)
    for (n, C, eps, mu, sig) in ((16, 37, 1e-5, 0.0, 1.0), (5, 768, 1e-5, 100.0, 0.01),
                                 (3, 1600, 1e-5, 0.0, 1.0), (4, 3, 0.5, 1.0, 2.0)):
        x = mu + sig * rng.normal(size=(n, C))
        w = 1.0 + 0.1 * rng.normal(size=C)
        b = 0.1 * rng.normal(size=C)
        dout = rng.normal(size=(n, C))
        tx = torch.tensor(x, dtype=torch.float64, requires_grad=True)
        tw = torch.tensor(w, dtype=torch.float64, requires_grad=True)
        tb = torch.tensor(b, dtype=torch.float64, requires_grad=True)
        ty = torch.nn.functional.layer_norm(tx, (C,), tw, tb, eps)
        ty.backward(torch.tensor(dout, dtype=torch.float64))
        out, mean, rstd = orc.forward(x, w, b, eps)
        dinp, dw, db = orc.backward(dout, x, w, mean, rstd)
        tol = 1e-12 if sig >= 1 else 1e-9    # torch's own rounding at var 1e-4
        assert _rel(out, ty.detach().numpy()) < tol, "torch forward"
        assert _rel(dinp, tx.grad.numpy()) < tol, "torch dinp"
        assert _rel(dw, tw.grad.numpy()) < tol, "torch dweight"
        assert _rel(db, tb.grad.numpy()) < 1e-13, "torch dbias"


def pin_rejects_bad_shapes(orc):
    """N < 0 and C <= 0 are rejected (the numpy wrapper cannot express N < 0,
    so an empty C is the case checked here); N = 0 is a valid empty batch."""
    import pytest
    with pytest.raises(ValueError):
        orc.forward(np.zeros((2, 0)), np.zeros(0), np.zeros(0), 1e-5)
    out, mean, rstd = orc.forward(np.zeros((0, 4)), np.ones(4), np.zeros(4), 1e-5)
    assert out.shape == (0, 4) and mean.shape == (0,)
    dinp, dw, db = orc.backward(np.zeros((0, 4)), np.zeros((0, 4)), np.ones(4),
                                np.zeros(0), np.zeros(0))
    assert np.array_equal(dw, np.zeros(4)) and np.array_equal(db, np.zeros(4))


# ----------------------------------------------------------- rounding pins

def _format_values(fmt):
    """Every positive finite value of a format, ascending, with its bit
    pattern (for fp32, only bf16 and f16 are enumerated: 2^31 values are too
    many; fp32 is pinned by numpy's cast and by local neighbourhoods)."""
    if fmt == "bf16":
        bits = np.arange(1, 0x7F80, dtype=np.uint32)
        vals = (bits << np.uint32(16)).view(np.float32).astype(np.float64)
    elif fmt == "f16":
        bits = np.arange(1, 0x7C00, dtype=np.uint16)
        vals = bits.view(np.float16).astype(np.float64)
        bits = bits.astype(np.uint32)
    else:
        raise ValueError(fmt)
    return vals, bits


def _brute_round(v, vals, bits):
    """Nearest of 0 and ``vals`` to the exact value v (Fraction or float), ties
    to the even bit pattern; beyond the largest value by half a spacing or
    more, infinity."""
    v = Fraction(v)
    sign = -1 if v < 0 else 1
    a = abs(v)
    top = Fraction(float(vals[-1]))
    half_top = (top - Fraction(float(vals[-2]))) / 2
    if a >= top + half_top:
        return sign * math.inf
    k = int(np.searchsorted(vals, float(a), side="right"))   # vals[k-1] <= a (about)
    cands = [(Fraction(0), 0)]
    for j in range(max(0, k - 2), min(len(vals), k + 2)):
        cands.append((Fraction(float(vals[j])), int(bits[j])))
    best = min(cands, key=lambda cb: (abs(cb[0] - a), cb[1] & 1))
    return sign * float(best[0])


def _probe_values(rng, lo_exp, hi_exp, n):
    """Random magnitudes over [2^lo_exp, 2^hi_exp), both signs."""
    e = rng.uniform(lo_exp, hi_exp, n)
    return np.where(rng.random(n) < 0.5, -1.0, 1.0) * np.exp2(e)


def pin_round_brute_force(orc):
    """oracle_round_format against brute force over every bfloat16 and fp16
    value: random values across the normal and subnormal ranges, exact ties
    (midpoints of neighbouring values) and the overflow boundary."""
    rng = _rng(21)
    for fmt, (lo, hi) in (("bf16", (-136.0, 128.5)), ("f16", (-26.0, 16.5))):
        vals, bits = _format_values(fmt)
        probes = list(_probe_values(rng, lo, hi, 400))
        idx = rng.integers(0, len(vals) - 1, 200)
        probes += [float((Fraction(float(vals[i])) + Fraction(float(vals[i + 1]))) / 2)
                   for i in idx]                                    # exact midpoints
        top, below = float(vals[-1]), float(vals[-2])
        probes += [top, top + (top - below) / 2, np.nextafter(top + (top - below) / 2, 0.0),
                   float(vals[0]) / 2, float(vals[0]) * 1.5, -float(vals[0]) / 2]
        got = orc.round_to(np.array(probes), fmt)
        for v, g in zip(probes, got):
            want = _brute_round(v, vals, bits)
            assert g == want or (math.isinf(want) and g == want), \
                f"{fmt}: round({v!r}) = {g!r}, brute force {want!r}"


def pin_round_numpy_casts(orc):
    """fp32 and fp16 rounding against numpy's float64 -> float32 / float16
    casts (IEEE round to nearest even), including fp32 ties built exactly
    as midpoints of neighbouring fp32 values and subnormals."""
    rng = _rng(22)
    v32 = _probe_values(rng, -155.0, 128.5, 20000)
    f = rng.normal(size=2000).astype(np.float32)
    mids = (f.astype(np.float64)
            + (np.nextafter(f, np.float32(np.inf)).astype(np.float64) - f.astype(np.float64)) / 2)
    v32 = np.concatenate([v32, mids, [3.4028235677973366e38, 3.40282357e38, 1e-46, -7e-46]])
    with np.errstate(over="ignore"):
        want32 = v32.astype(np.float32).astype(np.float64)
    got32 = orc.round_to(v32, "f32")
    assert np.array_equal(got32, want32), "fp32 rounding disagrees with numpy"
    v16 = _probe_values(rng, -27.0, 16.5, 20000)
    with np.errstate(over="ignore"):
        want16 = v16.astype(np.float16).astype(np.float64)
    assert np.array_equal(orc.round_to(v16, "f16"), want16), "fp16 rounding vs numpy"


def pin_residual_forward(orc):
    """forward_residual: x is the brute-force rounding of the exact sum
    resid + branch (bf16 operands), and with branch = 0 the whole result is
    the plain forward of resid."""
    rng = _rng(23)
    vals, bits = _format_values("bf16")
    n, C = 3, 11
    a = orc.round_to(rng.normal(size=(n, C)), "bf16")
    b = orc.round_to(rng.normal(scale=0.3, size=(n, C)) * np.exp2(rng.integers(-12, 4, (n, C))),
                     "bf16")
    w = 1.0 + 0.1 * rng.normal(size=C)
    bias = 0.1 * rng.normal(size=C)
    x, out, mean, rstd = orc.forward_residual(a, b, w, bias, 1e-5, "bf16")
    for i in range(n):
        for j in range(C):
            want = _brute_round(Fraction(float(a[i, j])) + Fraction(float(b[i, j])), vals, bits)
            assert x[i, j] == want, "residual sum rounding"
    o2, m2, s2 = orc.forward(x, w, bias, 1e-5)
    assert np.array_equal(out, o2) and np.array_equal(mean, m2) and np.array_equal(rstd, s2)
    x0, o0, m0, s0 = orc.forward_residual(a, np.zeros_like(a), w, bias, 1e-5, "bf16")
    o1, m1, s1 = orc.forward(a, w, bias, 1e-5)
    assert np.array_equal(x0, a), "x = resid when branch = 0"
    assert np.array_equal(o0, o1) and np.array_equal(m0, m1) and np.array_equal(s0, s1)


# -------------------------------------------------------- backward variants

def pin_backward_linearity(orc):
    """The gradient is linear in dout: accumulating the gradient of dout2
    onto that of dout1 gives the gradient of dout1 + dout2 (dinp, dweight and
    dbias), with saved and with recomputed statistics."""
    rng = _rng(24)
    n, C, eps = 6, 19, 1e-5
    x = rng.normal(size=(n, C))
    w = 1.0 + 0.1 * rng.normal(size=C)
    d1, d2 = rng.normal(size=(n, C)), rng.normal(size=(n, C))
    _, mean, rstd = orc.forward(x, w, np.zeros(C), eps)
    for recompute in (False, True):
        g1 = orc.backward_ex(d1, x, w, mean, rstd, eps, recompute=recompute)
        acc = orc.backward_ex(d2, x, w, mean, rstd, eps, dinp_prev=g1[0], dweight_prev=g1[1],
                              dbias_prev=g1[2], recompute=recompute)
        both = orc.backward(d1 + d2, x, w, mean, rstd)
        for got, want, name in zip(acc, both, ("dinp", "dweight", "dbias")):
            assert _rel(got, want) < 1e-12, f"accumulated {name} (recompute={recompute})"
    # accumulating only the parameters leaves dinp overwritten
    g = orc.backward_ex(d2, x, w, mean, rstd, eps, dweight_prev=np.ones(C), dbias_prev=np.ones(C))
    plain = orc.backward(d2, x, w, mean, rstd)
    assert _rel(g[0], plain[0]) < 1e-15 and _rel(g[1] - 1.0, plain[1]) < 1e-12


def pin_backward_recompute_torch(orc):
    """Recomputing the statistics: torch autograd of layer_norm in float64
    (which computes mean and rstd from the input itself), including rows whose
    variance is comparable to eps."""
    import torch
    rng = _rng(25)
    for (n, C, eps, mu, sig) in ((7, 33, 1e-5, 0.0, 1.0), (4, 768, 1e-5, 100.0, 0.01),
                                 (5, 64, 1e-5, 0.0, 2e-3)):
        x = mu + sig * rng.normal(size=(n, C))
        w = 1.0 + 0.1 * rng.normal(size=C)
        dout = rng.normal(size=(n, C))
        tx = torch.tensor(x, dtype=torch.float64, requires_grad=True)
        tw = torch.tensor(w, dtype=torch.float64, requires_grad=True)
        tb = torch.zeros(C, dtype=torch.float64, requires_grad=True)
        torch.nn.functional.layer_norm(tx, (C,), tw, tb, eps).backward(
            torch.tensor(dout, dtype=torch.float64))
        dinp, dw, db = orc.backward_ex(dout, x, w, None, None, eps, recompute=True)
        tol = 1e-12 if sig >= 1 else 1e-9
        assert _rel(dinp, tx.grad.numpy()) < tol, "recomputed dinp vs torch"
        assert _rel(dw, tw.grad.numpy()) < tol, "recomputed dweight vs torch"
        assert _rel(db, tb.grad.numpy()) < 1e-13, "recomputed dbias vs torch"


ALL_PINS = [pin_one_column, pin_two_columns, pin_constant_rows, pin_scale_by_two,
            pin_shift_invariance, pin_unit_affine_moments, pin_finite_differences,
            pin_row_identities, pin_dbias_integer_sum, pin_hand_worked,
            pin_torch_float64, pin_round_brute_force, pin_round_numpy_casts,
            pin_residual_forward, pin_backward_linearity, pin_backward_recompute_torch]
