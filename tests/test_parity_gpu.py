"""Parity of the CUDA library with the CPU oracle, element by element, on the
same seeded inputs (needs a B200)."""
import numpy as np
import pytest
import torch

import gpu_util as gu
import oracle
import tolerances as tol
from layernorm_fwd_bwd_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return gu.ln()


def _forward_parity(lib, batch, label, scaled=False):
    """scaled: judge against the magnitude of the summands (shapes outside
    the five workloads); otherwise each tensor's own max-abs."""
    w = batch.workload
    N, C, d = batch.inp.shape[0], w.C, w.dtype
    inp, wt, bs, dout = gu.batch_to_device(batch)
    out, mean, rstd = gu.forward(lib, inp, wt, bs, N, C, batch.eps, d)
    ref_out, ref_mean, ref_rstd = oracle.ln_forward(batch.f64("inp"), batch.f64("weight"),
                                                    batch.f64("bias"), batch.eps)
    sc = _scales(batch, ref_mean, ref_rstd) if scaled else {}
    res = [tol.check(f"{label} out", gu.to_f64(out), ref_out, d, "act_fwd"),
           tol.check(f"{label} mean", gu.to_f64(mean), ref_mean, d, "stats",
                     sc.get("mean", 0.0)),
           tol.check(f"{label} rstd", gu.to_f64(rstd), ref_rstd, d, "stats")]
    return (inp, wt, bs, dout), (out, mean, rstd), (ref_mean, ref_rstd), res


def _scales(batch, mean, rstd):
    return tol.magnitude_scales(batch.f64("inp"), batch.f64("dout"), batch.f64("weight"),
                                mean, rstd)


def _backward_parity(lib, batch, dev, label, ref_stats, scaled=False):
    """Backward as a function of its arguments: both sides get the same fp32
    mean/rstd (the oracle's statistics rounded to fp32)."""
    w = batch.workload
    N, C, d = batch.inp.shape[0], w.C, w.dtype
    inp, wt, _, dout = dev
    mean32 = ref_stats[0].astype(np.float32)
    rstd32 = ref_stats[1].astype(np.float32)
    dinp, dw, db = gu.backward(lib, dout, inp, wt, torch.from_numpy(mean32).cuda(),
                               torch.from_numpy(rstd32).cuda(), N, C, d)
    r_dinp, r_dw, r_db = oracle.ln_backward(batch.f64("dout"), batch.f64("inp"),
                                            batch.f64("weight"), mean32, rstd32)
    sc = _scales(batch, mean32, rstd32) if scaled else {}
    return [tol.check(f"{label} dinp", gu.to_f64(dinp), r_dinp, d, "act_bwd",
                      sc.get("dinp", 0.0)),
            tol.check(f"{label} dweight", gu.to_f64(dw), r_dw, d, "param_grad",
                      sc.get("dweight", 0.0)),
            tol.check(f"{label} dbias", gu.to_f64(db), r_db, d, "param_grad",
                      sc.get("dbias", 0.0))]


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_full_workload_parity(lib, name):
    """Every element of every output at the full workload sizes, in the launch
    configuration the benchmark uses: forward vs the oracle; backward as a
    function of its arguments (both sides get the oracle's statistics rounded
    to fp32); and, except for the stress workload, the GPU forward feeding the
    GPU backward against the oracle in double from end to end.  (In the stress
    workload the fp32 rounding of a mean near 100 alone moves xhat by up to
    rstd * ulp(100)/2 ~ 4e-4, so there the backward is judged only as a
    function of its own arguments.)"""
    batch = gu.full_batch(name)
    dev, (out, mean, rstd), ref_stats, res = _forward_parity(lib, batch, name)
    res += _backward_parity(lib, batch, dev, name, ref_stats)
    w = batch.workload
    if w.const_row_period:
        rows = np.arange(w.N) % w.const_row_period == 0
        # constant rows: deviations are exactly zero, so out == bias bitwise
        # and mean == the row's value bitwise
        out_h = gu.to_f64(out)[rows]
        assert np.array_equal(out_h, np.broadcast_to(batch.f64("bias"), out_h.shape))
        assert np.array_equal(gu.to_f64(mean)[rows], batch.f64("inp")[rows, 0])
    else:
        inp, wt, _, dout = dev
        dinp, dw, db = gu.backward(lib, dout, inp, wt, mean, rstd, w.N, w.C, w.dtype)
        r_dinp, r_dw, r_db = oracle.ln_backward(batch.f64("dout"), batch.f64("inp"),
                                                batch.f64("weight"), ref_stats[0],
                                                ref_stats[1])
        res += [tol.check(f"{name} chained dinp", gu.to_f64(dinp), r_dinp, w.dtype, "act_bwd"),
                tol.check(f"{name} chained dweight", gu.to_f64(dw), r_dw, w.dtype,
                          "param_grad"),
                tol.check(f"{name} chained dbias", gu.to_f64(db), r_db, w.dtype,
                          "param_grad")]
    print(res)


SWEEP_C = [1, 2, 3, 7, 8, 31, 33, 127, 128, 768, 1023, 1024, 1600, 2048, 2056, 4096,
           8192, 16384, 20000]


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("C", SWEEP_C)
@pytest.mark.parametrize("N", [1, 3, 257])
def test_shape_sweep(lib, dtype, C, N):
    """Ragged tails of the vector paths, every row-ownership variant, and the
    scalar path (C * size not a multiple of 16 bytes, or C past the vector
    limits)."""
    batch = wl.custom(dtype, N, C, seed=1000 + C + N)
    dev, _, ref_stats, _ = _forward_parity(lib, batch, f"{dtype} {N}x{C}", scaled=True)
    _backward_parity(lib, batch, dev, f"{dtype} {N}x{C}", ref_stats, scaled=True)


# Widths around and inside the split backward (16-bit rows of 7..8 vectors per
# row-warp lane, row and column warps on one ring; narrower rows take the
# rings next to it): column slices that end inside a warp and rings of 3 and 4
# stages.  N = 7 is one partial tile; N = 5003 gives each block about four
# tiles of 8 rows and a last tile of 3.
SPLIT_C = [1032, 1184, 1192, 1416, 1536, 1760, 1784, 1800, 2040]


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("C", SPLIT_C)
@pytest.mark.parametrize("N", [7, 5003])
def test_split_backward_widths(lib, dtype, C, N):
    batch = wl.custom(dtype, N, C, seed=5000 + C + N, dout_sigma=0.02)
    dev, _, ref_stats, _ = _forward_parity(lib, batch, f"{dtype} {N}x{C}", scaled=True)
    _backward_parity(lib, batch, dev, f"{dtype} {N}x{C}", ref_stats, scaled=True)


# Forward rows of 17..32 vectors per lane on four warps per row (16-bit C =
# 4104..8192, fp32 C = 2052..4096), one to three tiles per block; N = 5 is one
# partial tile, N = 1003 several blocks with a ragged last one.
FOUR_C = {"bf16": [4104, 5008, 6144, 8192], "f16": [4104, 8192], "f32": [2056, 3000, 4096]}


@pytest.mark.parametrize("dtype,C", [(d, c) for d, cs in FOUR_C.items() for c in cs])
@pytest.mark.parametrize("N", [5, 1003])
def test_four_warp_forward_widths(lib, dtype, C, N):
    batch = wl.custom(dtype, N, C, seed=7000 + C + N)
    dev, _, ref_stats, _ = _forward_parity(lib, batch, f"{dtype} {N}x{C}", scaled=True)
    _backward_parity(lib, batch, dev, f"{dtype} {N}x{C}", ref_stats, scaled=True)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_widest_row(lib, dtype):
    """C = LN_MAX_C (2^24 channels, 32 or 64 MB a row), two rows, every
    element: rows past every vectorised variant take the scalar kernels with
    one block per row, and the backward's workspace bound leaves it two
    blocks."""
    C = lib.LN_MAX_C
    batch = wl.custom(dtype, 2, C, seed=24)
    label = f"{dtype} 2x{C}"
    dev, _, ref_stats, res = _forward_parity(lib, batch, label, scaled=True)
    res += _backward_parity(lib, batch, dev, label, ref_stats, scaled=True)
    print(res)


# (dtype, C, rows of one period P, periods k): N * C = k * P * C > 2^31
BEYOND_INT32 = [("bf16", 768, 4096, 700),    # tile forward, ring backward
                ("f32", 768, 4096, 700),     # the same kernels, 8.8 GB arrays
                ("bf16", 770, 4096, 700),    # scalar kernels (C * 2 not a multiple of 16)
                ("bf16", 4096, 1024, 520),   # two-warp tile forward, six-warp ring backward
                ("bf16", 16000, 256, 560),   # register-resident kernels, 16 warps per row
                ("bf16", 1600, 4096, 330),   # split backward (row and column warps)
                ("bf16", 8192, 256, 1030)]   # four-warp tile forward, register-resident backward


@pytest.mark.parametrize("dtype,C,P,k", BEYOND_INT32)
def test_beyond_int32_elements(lib, dtype, C, P, k):
    """More than 2^31 elements per array (element and byte offsets past 32
    bits).  The rows repeat with period P (the first P rows copied k times on
    the device), which fixes the result at any size: every output row equals
    the same row of the first period bit for bit, the first period matches
    the oracle, and dweight/dbias equal k times the first period's oracle
    sums.  The backward gets the oracle's statistics rounded to fp32."""
    N = P * k
    assert N * C > 2 ** 31
    batch = wl.custom(dtype, P, C, seed=2 ** 31 + C, dout_sigma=0.02)
    inp_p, wt, bs, dout_p = gu.batch_to_device(batch)
    ref_out, ref_mean, ref_rstd = oracle.ln_forward(batch.f64("inp"), batch.f64("weight"),
                                                    batch.f64("bias"), batch.eps)
    m32, r32 = ref_mean.astype(np.float32), ref_rstd.astype(np.float32)
    r_dinp, r_dw, r_db = oracle.ln_backward(batch.f64("dout"), batch.f64("inp"),
                                            batch.f64("weight"), m32, r32)
    sc = _scales(batch, m32, r32)

    def periodic(name, t):
        b = gu.bits(t).reshape(k, -1)
        for a in range(0, k, 64):
            assert bool((b[a:a + 64] == b[0]).all()), f"{name}: period {a}.. differs"

    label = f"{dtype} {N}x{C}"
    inp = inp_p.repeat(k, 1)
    out, mean, rstd = gu.forward(lib, inp, wt, bs, N, C, batch.eps, dtype)
    for name, t in (("out", out), ("mean", mean), ("rstd", rstd)):
        periodic(name, t)
    res = [tol.check(f"{label} out", gu.to_f64(out[:P]), ref_out, dtype, "act_fwd"),
           tol.check(f"{label} mean", gu.to_f64(mean[:P]), ref_mean, dtype, "stats",
                     sc["mean"]),
           tol.check(f"{label} rstd", gu.to_f64(rstd[:P]), ref_rstd, dtype, "stats")]
    del out
    dout = dout_p.repeat(k, 1)
    dinp, dw, db = gu.backward(lib, dout, inp, wt, torch.from_numpy(m32).cuda().repeat(k),
                               torch.from_numpy(r32).cuda().repeat(k), N, C, dtype)
    periodic("dinp", dinp)
    res += [tol.check(f"{label} dinp", gu.to_f64(dinp[:P]), r_dinp, dtype, "act_bwd",
                      sc["dinp"]),
            tol.check(f"{label} dweight", gu.to_f64(dw), k * r_dw, dtype, "param_grad",
                      k * sc["dweight"]),
            tol.check(f"{label} dbias", gu.to_f64(db), k * r_db, dtype, "param_grad",
                      k * sc["dbias"])]
    assert lib.device_status() == 0
    print(res)
    del inp, dout, dinp, mean, rstd
    torch.cuda.empty_cache()


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("C", [768, 1600, 5])
def test_misaligned_pointers(lib, dtype, C):
    """Arrays that start one element past a 16-byte boundary take the scalar
    path and give the same results."""
    N = 37
    batch = wl.custom(dtype, N, C, seed=77)
    td = gu.TORCH_DT[dtype]

    def shifted(a):
        t = gu.to_device(a.reshape(-1), dtype)
        buf = torch.empty(t.numel() + 1, dtype=td, device="cuda")
        buf[1:] = t
        return buf[1:]

    inp, wt, bs, dout = (shifted(batch.inp), shifted(batch.weight), shifted(batch.bias),
                         shifted(batch.dout))
    assert inp.data_ptr() % 16 != 0
    outb = torch.empty(N * C + 1, dtype=td, device="cuda")
    out = outb[1:]
    mean = torch.empty(N, device="cuda")
    rstd = torch.empty(N, device="cuda")
    lib.ln_forward(out, mean, rstd, inp, wt, bs, N, C, batch.eps, gu.DT[dtype])
    ro, rm, rr = oracle.ln_forward(batch.f64("inp"), batch.f64("weight"),
                                   batch.f64("bias"), batch.eps)
    m32, r32 = rm.astype(np.float32), rr.astype(np.float32)
    sc = _scales(batch, m32, r32)
    tol.check("out", gu.to_f64(out).reshape(N, C), ro, dtype, "act_fwd")
    tol.check("mean", gu.to_f64(mean), rm, dtype, "stats", sc["mean"])
    dinpb = torch.empty(N * C + 1, dtype=td, device="cuda")
    dw = torch.empty(C, device="cuda")
    db = torch.empty(C, device="cuda")
    lib.ln_backward(dinpb[1:], dw, db, dout, inp, wt, torch.from_numpy(m32).cuda(),
                    torch.from_numpy(r32).cuda(), N, C, gu.DT[dtype])
    rd, rw, rb = oracle.ln_backward(batch.f64("dout"), batch.f64("inp"),
                                    batch.f64("weight"), m32, r32)
    tol.check("dinp", gu.to_f64(dinpb[1:]).reshape(N, C), rd, dtype, "act_bwd", sc["dinp"])
    tol.check("dweight", gu.to_f64(dw), rw, dtype, "param_grad", sc["dweight"])
    tol.check("dbias", gu.to_f64(db), rb, dtype, "param_grad", sc["dbias"])


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("C", [768, 1600, 7, 20000])
def test_guard_regions_and_full_coverage(lib, dtype, C):
    """Outputs sit inside larger buffers whose margins hold a sentinel; after
    both calls the margins are unchanged and no output element is left at
    its NaN pre-fill."""
    N = 130
    G = 256                       # margin elements on each side (keeps 16-B alignment)
    batch = wl.custom(dtype, N, C, seed=5)
    inp, wt, bs, dout = gu.batch_to_device(batch)
    td = gu.TORCH_DT[dtype]

    def guarded(n, tdt):
        buf = torch.full((n + 2 * G,), float("nan"), dtype=tdt, device="cuda")
        buf[:G] = 3.25
        buf[-G:] = -7.5
        return buf, buf[G:G + n]

    def intact(buf):
        return bool((buf[:G] == 3.25).all()) and bool((buf[-G:] == -7.5).all())

    ob, out = guarded(N * C, td)
    mb, mean = guarded(N, torch.float32)
    rb_, rstd = guarded(N, torch.float32)
    lib.ln_forward(out, mean, rstd, inp, wt, bs, N, C, batch.eps, gu.DT[dtype])
    db_, dinp = guarded(N * C, td)
    wb, dw = guarded(C, torch.float32)
    bb, dbias = guarded(C, torch.float32)
    lib.ln_backward(dinp, dw, dbias, dout, inp, wt, mean, rstd, N, C, gu.DT[dtype])
    torch.cuda.synchronize()
    for name, buf, view in (("out", ob, out), ("mean", mb, mean), ("rstd", rb_, rstd),
                            ("dinp", db_, dinp), ("dweight", wb, dw), ("dbias", bb, dbias)):
        assert intact(buf), f"{name}: write outside its bounds"
        assert not bool(torch.isnan(view.float()).any()), f"{name}: element not written"


@pytest.mark.parametrize("name", ["gpt2_124m_bf16", "stress_fp32_65536x768"])
def test_deterministic(lib, name):
    """Same inputs, different launch histories: bitwise-identical outputs."""
    w = wl.WORKLOADS[name]
    batch = wl.generate(w, rows=np.arange(8192))
    inp, wt, bs, dout = gu.batch_to_device(batch)
    N = 8192
    results = []
    for k in range(3):
        if k == 1:   # perturb: an unrelated call of another shape in between
            other = wl.custom(w.dtype, 999, 1600, seed=3)
            oi, ow, ob, od = gu.batch_to_device(other)
            gu.forward(lib, oi, ow, ob, 999, 1600, 1e-5, w.dtype)
        stream = torch.cuda.Stream() if k == 2 else torch.cuda.current_stream()
        stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(stream):
            out, mean, rstd = gu.forward(lib, inp, wt, bs, N, w.C, batch.eps, w.dtype)
            dinp, dw, db = gu.backward(lib, dout, inp, wt, mean, rstd, N, w.C, w.dtype)
        torch.cuda.synchronize()
        results.append([t.clone() for t in (out, mean, rstd, dinp, dw, db)])
    def bits(t):
        return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)

    for r in results[1:]:
        for a, b in zip(results[0], r):
            assert torch.equal(bits(a), bits(b))


# (dtype, N, C of the first and third call, C of the second): one kernel
# instantiation each, whose dynamic shared memory grows with C.  The second C
# appears in no other test, so its first call always sets up that kernel at a
# smaller size after the larger one.
SHRINK_GROW = [("bf16", 64, 16384, 15992),   # register-resident forward, 16 warps per row
               ("bf16", 4096, 768, 648),     # tile forward, one-warp ring backward
               ("f32", 2048, 2560, 2440),    # fp32 ring backward, shared rows
               ("bf16", 1024, 4096, 3976)]   # two-warp tile forward, wide backward


@pytest.mark.parametrize("dtype,N,C_big,C_small", SHRINK_GROW)
def test_shapes_shrinking_then_growing(lib, dtype, N, C_big, C_small):
    """A kernel's dynamic shared-memory limit is one value per kernel and
    device: a call at a smaller C must not leave a limit that a later call
    at the larger C, whose set-up was cached, launches above.  Every call
    returns LN_OK and matches the oracle."""
    for C in (C_big, C_small, C_big):
        batch = wl.custom(dtype, N, C, seed=3000 + C)
        label = f"{dtype} {N}x{C}"
        dev, _, ref_stats, _ = _forward_parity(lib, batch, label, scaled=True)
        _backward_parity(lib, batch, dev, label, ref_stats, scaled=True)


def test_workspace_refusal_launches_nothing(lib):
    """LN_ERR_WORKSPACE: a backward whose partial sums exceed the device's
    workspace cap is refused before any launch, leaves the outputs and the
    CUDA context untouched, and the next call within the cap succeeds."""
    N, C = 4096, 768
    batch = wl.custom("bf16", N, C, seed=31)
    inp, wt, bs, dout = gu.batch_to_device(batch)
    _, mean, rstd = gu.forward(lib, inp, wt, bs, N, C, batch.eps, "bf16")
    want = gu.backward(lib, dout, inp, wt, mean, rstd, N, C, "bf16")
    torch.cuda.synchronize()
    dinp = gu.nan_tensor((N, C), torch.bfloat16)
    dw = gu.nan_tensor((C,), torch.float32)
    db = gu.nan_tensor((C,), torch.float32)
    try:
        lib.set_workspace_limit(2 * C * 4 - 1)        # less than one block's partial row
        before = lib.launch_count()
        for call in (lambda: lib.ln_backward(dinp, dw, db, dout, inp, wt, mean, rstd, N, C,
                                             lib.LN_BF16),
                     lambda: lib.ln_backward_ex(dinp, dw, db, dout, inp, wt, None, None, N, C,
                                                batch.eps, lib.LN_BF16,
                                                lib.LN_BWD_RECOMPUTE_STATS)):
            with pytest.raises(lib.LNError) as e:
                call()
            assert e.value.status == lib.LN_ERR_WORKSPACE
        assert lib.launch_count() == before
        torch.cuda.synchronize()                          # no error left behind
        assert bool(torch.isnan(dinp.float()).all()) and bool(torch.isnan(dw).all())
        # the allocation-free entry point does not draw from the pool
        lib.ln_backward_noalloc(dinp, dw, db, dout, inp, wt, mean, rstd, N, C, lib.LN_BF16)
        torch.cuda.synchronize()
        assert lib.launch_count() == before + 2
    finally:
        lib.set_workspace_limit(0)
    got = gu.backward(lib, dout, inp, wt, mean, rstd, N, C, "bf16")
    torch.cuda.synchronize()
    for g, r in zip(got, want):
        assert bool((gu.bits(g) == gu.bits(r)).all())
    assert lib.device_status() == 0


def test_empty_batch(lib):
    C = 64
    w = torch.ones(C, device="cuda")
    dw = torch.full((C,), float("nan"), device="cuda")
    db = torch.full((C,), float("nan"), device="cuda")
    before = lib.launch_count()
    lib.ln_forward(None, None, None, None, w, w, 0, C, 1e-5, 0)
    lib.ln_backward(None, dw, db, None, None, w, None, None, 0, C, 0)
    torch.cuda.synchronize()
    assert lib.launch_count() == before
    assert bool((dw == 0).all()) and bool((db == 0).all())


def test_errors_launch_nothing(lib):
    x = torch.zeros(4, 8, device="cuda")
    v = torch.zeros(8, device="cuda")
    s = torch.zeros(4, device="cuda")
    before = lib.launch_count()
    for args, status in (
            ((None, s, s, x, v, v, 4, 8, 1e-5, 0), lib.LN_ERR_NULL),
            ((x, s, s, x, v, None, 4, 8, 1e-5, 0), lib.LN_ERR_NULL),
            ((x, s, s, x, v, v, 4, 8, 1e-5, 5), lib.LN_ERR_DTYPE),
            ((x, s, s, x, v, v, 4, 8, float("nan"), 0), lib.LN_ERR_EPS),
            ((x, s, s, x, v, v, -4, 8, 1e-5, 0), lib.LN_ERR_SHAPE)):
        with pytest.raises(lib.LNError) as e:
            lib.ln_forward(*args)
        assert e.value.status == status
    with pytest.raises(lib.LNError) as e:
        lib.ln_backward(x, v, v, x, x, v, s, None, 4, 8, 0)
    assert e.value.status == lib.LN_ERR_NULL
    assert lib.launch_count() == before


def test_launch_counts(lib):
    """One forward launches one kernel; one backward two (row pass, column
    finalise)."""
    batch = wl.custom("bf16", 64, 768, seed=9)
    inp, wt, bs, dout = gu.batch_to_device(batch)
    c0 = lib.launch_count()
    out, mean, rstd = gu.forward(lib, inp, wt, bs, 64, 768, 1e-5, "bf16")
    c1 = lib.launch_count()
    gu.backward(lib, dout, inp, wt, mean, rstd, 64, 768, "bf16")
    c2 = lib.launch_count()
    assert (c1 - c0, c2 - c1) == (1, 2)


def test_repeated_runs_bitwise_identical(lib):
    """Twenty forward+backward passes over the full GPT-2 124M workload give
    bitwise-identical outputs.  A race between the warps reading a shared
    memory stage and a bulk copy refilling it shows up here as rows that
    differ from one run to the next."""
    w = wl.WORKLOADS["gpt2_124m_bf16"]
    batch = gu.full_batch(w.name)
    inp, wt, bs, dout = gu.batch_to_device(batch)
    first = None
    for _ in range(20):
        out, mean, rstd = gu.forward(lib, inp, wt, bs, w.N, w.C, batch.eps, w.dtype)
        dinp, dw, db = gu.backward(lib, dout, inp, wt, mean, rstd, w.N, w.C, w.dtype)
        cur = [out.view(torch.int16), mean.view(torch.int32), rstd.view(torch.int32),
               dinp.view(torch.int16), dw.view(torch.int32), db.view(torch.int32)]
        if first is None:
            first = [t.clone() for t in cur]
        else:
            for a, b in zip(first, cur):
                assert torch.equal(a, b)
    assert lib.device_status() == 0


def test_fp16_gpt2_124m_shape(lib):
    """fp16 activations at the GPT-2 124M LayerNorm shape (65536 x 768,
    the bf16 workload's distributions), every element: forward, backward as a
    function of its arguments, and the forward feeding the backward."""
    batch = wl.custom("f16", 65536, 768, seed=20240530, dout_sigma=0.02)
    dev, (out, mean, rstd), ref_stats, res = _forward_parity(lib, batch, "f16 65536x768")
    res += _backward_parity(lib, batch, dev, "f16 65536x768", ref_stats)
    inp, wt, _, dout = dev
    dinp, dw, db = gu.backward(lib, dout, inp, wt, mean, rstd, 65536, 768, "f16")
    r = oracle.ln_backward(batch.f64("dout"), batch.f64("inp"), batch.f64("weight"),
                           ref_stats[0], ref_stats[1])
    res += [tol.check("f16 chained dinp", gu.to_f64(dinp), r[0], "f16", "act_bwd"),
            tol.check("f16 chained dweight", gu.to_f64(dw), r[1], "f16", "param_grad"),
            tol.check("f16 chained dbias", gu.to_f64(db), r[2], "f16", "param_grad")]
    print(res)


def test_cuda_graph_capture_replays_bitwise(lib):
    """A step (forward, backward, and an accumulating backward with
    recomputed statistics) captured in a CUDA graph and replayed gives the
    same bits as the eager calls: every launch is stream-ordered (the
    backward's workspace comes from a stream-ordered pool, so capture turns it
    into graph allocation nodes) and deterministic."""
    batch = wl.custom("bf16", 4096, 768, seed=77, dout_sigma=0.02)
    N, C, d = 4096, 768, "bf16"
    inp, wt, bs, dout = gu.batch_to_device(batch)
    td = gu.TORCH_DT[d]
    o = dict(out=torch.empty(N, C, dtype=td, device="cuda"),
             mean=torch.empty(N, device="cuda"), rstd=torch.empty(N, device="cuda"),
             dinp=torch.empty(N, C, dtype=td, device="cuda"),
             dw=torch.empty(C, device="cuda"), db=torch.empty(C, device="cuda"),
             dinp2=torch.empty(N, C, dtype=td, device="cuda"),
             dw2=torch.empty(C, device="cuda"), db2=torch.empty(C, device="cuda"))
    flags = lib.LN_BWD_ACCUMULATE_DINP | lib.LN_BWD_ACCUMULATE_DPARAMS | lib.LN_BWD_RECOMPUTE_STATS

    def step(stream):
        lib.ln_forward(o["out"], o["mean"], o["rstd"], inp, wt, bs, N, C, batch.eps,
                       gu.DT[d], stream)
        lib.ln_backward(o["dinp"], o["dw"], o["db"], dout, inp, wt, o["mean"], o["rstd"], N,
                        C, gu.DT[d], stream)
        o["dinp2"].copy_(o["dinp"])
        o["dw2"].copy_(o["dw"])
        o["db2"].copy_(o["db"])
        lib.ln_backward_ex(o["dinp2"], o["dw2"], o["db2"], dout, inp, wt, None, None, N, C,
                           batch.eps, gu.DT[d], flags, stream)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step(s)                                    # eager (also warms the library up)
    torch.cuda.synchronize()
    eager = {k: gu.bits(v).clone() for k, v in o.items()}
    for v in o.values():
        v.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(s)
    for _ in range(2):
        for v in o.values():
            v.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for k, v in o.items():
            assert torch.equal(gu.bits(v), eager[k]), f"graph replay: {k} differs"
    assert lib.device_status() == 0


def test_aliased_outputs_refused(lib):
    """In-place calls the header forbids raise LN_ERR_ALIAS and launch
    nothing: out == inp, dinp == dout, resid_out == resid."""
    N, C = 64, 768
    x = torch.randn(N, C, device="cuda").to(torch.bfloat16)
    w = torch.ones(C, device="cuda", dtype=torch.bfloat16)
    m = torch.empty(N, device="cuda")
    r = torch.empty(N, device="cuda")
    dw = torch.empty(C, device="cuda")
    n0 = lib.launch_count()
    with pytest.raises(lib.LNError) as e:
        lib.ln_forward(x, m, r, x, w, w, N, C, 1e-5, lib.LN_BF16)
    assert e.value.status == lib.LN_ERR_ALIAS
    with pytest.raises(lib.LNError) as e:
        lib.ln_backward(x, dw, dw.clone(), x, x.clone(), w, m, r, N, C, lib.LN_BF16)
    assert e.value.status == lib.LN_ERR_ALIAS
    with pytest.raises(lib.LNError) as e:
        lib.ln_forward_residual(x, x.clone(), m, r, x, x.clone(), w, w, N, C, 1e-5, lib.LN_BF16)
    assert e.value.status == lib.LN_ERR_ALIAS
    # outputs that overlap each other: mean == rstd; dweight == dbias
    y = torch.empty_like(x)
    with pytest.raises(lib.LNError) as e:
        lib.ln_forward(y, m, m, x, w, w, N, C, 1e-5, lib.LN_BF16)
    assert e.value.status == lib.LN_ERR_ALIAS
    with pytest.raises(lib.LNError) as e:
        lib.ln_backward(y, dw, dw, x, x.clone(), w, m, r, N, C, lib.LN_BF16)
    assert e.value.status == lib.LN_ERR_ALIAS
    assert lib.launch_count() == n0


def test_concurrent_host_threads(lib):
    """Several host threads call the library at once, on their own streams,
    as the first calls of a fresh process (so the per-device set-up, the
    kernels' shared-memory limits and the occupancy cache fill concurrently),
    on widths that reach the one-warp, two-warp, shared-row, split and fp32
    kernels.  Every output equals the same calls made afterwards from one
    thread, bit for bit; no call fails; no bounded wait ran out."""
    import json
    import os
    import subprocess
    import sys
    script = os.path.join(os.path.dirname(os.path.abspath(__file__)), "threads_check.py")
    proc = subprocess.run([sys.executable, script], capture_output=True, text=True,
                          timeout=600)
    assert proc.returncode == 0, proc.stderr[-3000:]
    res = json.loads([l for l in proc.stdout.splitlines() if l.startswith("{")][-1])
    assert res["errors"] == [], res["errors"]
    assert res["mismatches"] == [], res["mismatches"]
    assert res["device_status"] == 0
    # per thread and round: forward 1 launch, each backward 2
    assert res["threaded_launches"] == 6 * 12 * 5
