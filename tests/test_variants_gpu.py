"""Parity of the library's variants with the CPU oracle (needs a B200):
ln_forward_residual (x = resid + branch rounded to the dtype, then the
forward of x) and ln_backward_ex (accumulating dinp and/or dweight/dbias,
recomputing mean/rstd from inp).  Inputs come from the same seeded
generators as the plain tests; the variants' extra inputs (the branch, the
previous gradients) from ``workloads.generate_extras``."""
import numpy as np
import pytest
import torch

import gpu_util as gu
import oracle
import tolerances as tol
from layernorm_fwd_bwd_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ACC_DINP, ACC_PARAMS, RECOMPUTE = 1, 2, 4
FLAG_SETS = {"acc": ACC_DINP | ACC_PARAMS, "recompute": RECOMPUTE,
             "acc_recompute": ACC_DINP | ACC_PARAMS | RECOMPUTE,
             "acc_params_only": ACC_PARAMS, "acc_dinp_recompute": ACC_DINP | RECOMPUTE}


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return gu.ln()


def _fmt(dtype):
    return dtype          # the oracle's format names match the dtype names


def _residual(lib, batch, extras, label, scaled=False):
    w = batch.workload
    N, C, d = batch.inp.shape[0], w.C, w.dtype
    resid = gu.to_device(batch.inp, d)
    branch = gu.to_device(extras.branch, d)
    wt, bs = gu.to_device(batch.weight, d), gu.to_device(batch.bias, d)
    x = gu.nan_tensor((N, C), gu.TORCH_DT[d])
    out, mean, rstd = gu.forward_outputs(N, C, d)
    lib.ln_forward_residual(x, out, mean, rstd, resid, branch, wt, bs, N, C, batch.eps, gu.DT[d])
    rx, rout, rmean, rrstd = oracle.default().forward_residual(
        batch.f64("inp"), extras.f64("branch"), batch.f64("weight"), batch.f64("bias"),
        batch.eps, _fmt(d))
    # the rounded sum is bit-exact: both sides round the same exact sum once
    gx = gu.to_f64(x)
    assert np.array_equal(gx, rx), f"{label}: residual sum differs in " \
        f"{int(np.sum(gx != rx))} of {gx.size} elements"
    sc = tol.magnitude_scales(rx, batch.f64("dout"), batch.f64("weight"), rmean, rrstd) \
        if scaled else {}
    res = [tol.check(f"{label} out", gu.to_f64(out), rout, d, "act_fwd"),
           tol.check(f"{label} mean", gu.to_f64(mean), rmean, d, "stats", sc.get("mean", 0.0)),
           tol.check(f"{label} rstd", gu.to_f64(rstd), rrstd, d, "stats")]
    # the fused call normalises exactly the x it wrote: the plain forward of
    # resid_out gives the same bits
    out2, mean2, rstd2 = gu.forward(lib, x, wt, bs, N, C, batch.eps, d)
    for a, b, n in ((out, out2, "out"), (mean, mean2, "mean"), (rstd, rstd2, "rstd")):
        assert torch.equal(gu.bits(a), gu.bits(b)), \
            f"{label}: fused {n} differs from ln_forward(resid_out)"
    return res


def _backward_ex(lib, batch, extras, flags, label, scaled=False):
    w = batch.workload
    N, C, d = batch.inp.shape[0], w.C, w.dtype
    orc = oracle.default()
    inp, wt, _, dout = gu.batch_to_device(batch)
    recompute = bool(flags & RECOMPUTE)
    # saved statistics: the oracle's, rounded to fp32, given to both sides
    _, m64, s64 = orc.forward(batch.f64("inp"), batch.f64("weight"), batch.f64("bias"), batch.eps)
    mean32, rstd32 = m64.astype(np.float32), s64.astype(np.float32)
    mean_d = None if recompute else torch.from_numpy(mean32).cuda()
    rstd_d = None if recompute else torch.from_numpy(rstd32).cuda()
    if flags & ACC_DINP:
        dinp = gu.to_device(extras.dinp_prev, d)
    else:
        dinp = gu.nan_tensor((N, C), gu.TORCH_DT[d])
    if flags & ACC_PARAMS:
        dw = torch.from_numpy(extras.dweight_prev.copy()).cuda()
        db = torch.from_numpy(extras.dbias_prev.copy()).cuda()
    else:
        dw = gu.nan_tensor((C,), torch.float32)
        db = gu.nan_tensor((C,), torch.float32)
    lib.ln_backward_ex(dinp, dw, db, dout, inp, wt, mean_d, rstd_d, N, C, batch.eps, gu.DT[d],
                       flags)
    r_dinp, r_dw, r_db = orc.backward_ex(
        batch.f64("dout"), batch.f64("inp"), batch.f64("weight"),
        None if recompute else mean32, None if recompute else rstd32, batch.eps,
        dinp_prev=extras.f64("dinp_prev") if flags & ACC_DINP else None,
        dweight_prev=extras.f64("dweight_prev") if flags & ACC_PARAMS else None,
        dbias_prev=extras.f64("dbias_prev") if flags & ACC_PARAMS else None,
        recompute=recompute)
    sc = {}
    if scaled:
        sm, ss = (m64, s64) if recompute else (mean32, rstd32)
        sc = tol.magnitude_scales(batch.f64("inp"), batch.f64("dout"), batch.f64("weight"),
                                  sm, ss)
    return [tol.check(f"{label} dinp", gu.to_f64(dinp), r_dinp, d, "act_bwd",
                      sc.get("dinp", 0.0)),
            tol.check(f"{label} dweight", gu.to_f64(dw), r_dw, d, "param_grad",
                      sc.get("dweight", 0.0)),
            tol.check(f"{label} dbias", gu.to_f64(db), r_db, d, "param_grad",
                      sc.get("dbias", 0.0))]


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_residual_forward_full(lib, name):
    """Every element at the full workload sizes: the residual sum bit-exact,
    out/mean/rstd within the forward tolerances."""
    batch = gu.full_batch(name)
    extras = gu.full_extras(name)
    print(_residual(lib, batch, extras, name))


@pytest.mark.parametrize("flags", list(FLAG_SETS), ids=list(FLAG_SETS))
@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_backward_variants_full(lib, name, flags):
    """Every element at the full workload sizes.  Recomputing: the oracle's
    statistics in double feed its backward (the GPU recomputes its own in
    fp32, pivot-shifted), so this also covers the cancellation stress rows."""
    batch = gu.full_batch(name)
    extras = gu.full_extras(name)
    print(_backward_ex(lib, batch, extras, FLAG_SETS[flags], f"{name} {flags}"))


SWEEP_C = [1, 3, 8, 33, 128, 512, 768, 1024, 1600, 2056, 3072, 4096, 6144, 8192, 20000]


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("C", SWEEP_C)
@pytest.mark.parametrize("N", [1, 257])
def test_variant_sweep(lib, dtype, C, N):
    """Every kernel path of each variant (one-warp and shared-row rings with
    three arrays per stage, register-resident wide rows, scalar tails) with
    ragged tails."""
    batch = wl.custom(dtype, N, C, seed=3000 + C + N)
    extras = wl.generate_extras(batch.workload)
    label = f"{dtype} {N}x{C}"
    _residual(lib, batch, extras, label, scaled=True)
    for fl in ("acc", "recompute", "acc_recompute"):
        _backward_ex(lib, batch, extras, FLAG_SETS[fl], f"{label} {fl}", scaled=True)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("C", [1032, 1800, 2040])
@pytest.mark.parametrize("N", [7, 5003])
def test_split_accumulate_widths(lib, dtype, C, N):
    """The split backward with three arrays per stage (dinp accumulated) on
    partial and multi-tile blocks, and the recomputing backward at the same
    widths (the shared-row ring)."""
    batch = wl.custom(dtype, N, C, seed=6000 + C + N, dout_sigma=0.02)
    extras = wl.generate_extras(batch.workload)
    label = f"{dtype} {N}x{C}"
    for fl in ("acc", "acc_params_only", "recompute"):
        _backward_ex(lib, batch, extras, FLAG_SETS[fl], f"{label} {fl}", scaled=True)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("C", [768, 1600, 5])
def test_variants_misaligned(lib, dtype, C):
    """Arrays one element past a 16-byte boundary take the scalar kernels."""
    N = 37
    batch = wl.custom(dtype, N, C, seed=4000 + C)
    extras = wl.generate_extras(batch.workload)
    d = dtype
    td = gu.TORCH_DT[d]
    orc = oracle.default()

    def shifted(a):
        t = gu.to_device(a, d).reshape(-1)
        buf = torch.empty(t.numel() + 1, dtype=td, device="cuda")
        buf[1:] = t
        return buf[1:]

    resid, branch = shifted(batch.inp), shifted(extras.branch)
    wt, bs = shifted(batch.weight), shifted(batch.bias)
    x = torch.empty(N * C + 1, dtype=td, device="cuda")[1:]
    out = torch.empty(N * C + 1, dtype=td, device="cuda")[1:]
    mean = torch.empty(N, device="cuda")
    rstd = torch.empty(N, device="cuda")
    lib.ln_forward_residual(x, out, mean, rstd, resid, branch, wt, bs, N, C, batch.eps, gu.DT[d])
    rx, rout, rmean, rrstd = orc.forward_residual(batch.f64("inp"), extras.f64("branch"),
                                                  batch.f64("weight"), batch.f64("bias"),
                                                  batch.eps, _fmt(d))
    assert np.array_equal(gu.to_f64(x).reshape(N, C), rx)
    sc = tol.magnitude_scales(rx, batch.f64("dout"), batch.f64("weight"), rmean, rrstd)
    tol.check("misaligned residual out", gu.to_f64(out).reshape(N, C), rout, d, "act_fwd")
    tol.check("misaligned residual mean", gu.to_f64(mean), rmean, d, "stats", sc["mean"])
    dout, inp = shifted(batch.dout), shifted(batch.inp)
    dinp = shifted(extras.dinp_prev)
    dw = torch.from_numpy(extras.dweight_prev.copy()).cuda()
    db = torch.from_numpy(extras.dbias_prev.copy()).cuda()
    lib.ln_backward_ex(dinp, dw, db, dout, inp, wt, None, None, N, C, batch.eps, gu.DT[d],
                       ACC_DINP | ACC_PARAMS | RECOMPUTE)
    r = orc.backward_ex(batch.f64("dout"), batch.f64("inp"), batch.f64("weight"), None, None,
                        batch.eps, extras.f64("dinp_prev"), extras.f64("dweight_prev"),
                        extras.f64("dbias_prev"), recompute=True)
    _, m64, s64 = orc.forward(batch.f64("inp"), batch.f64("weight"), batch.f64("bias"), batch.eps)
    sc = tol.magnitude_scales(batch.f64("inp"), batch.f64("dout"), batch.f64("weight"), m64, s64)
    tol.check("misaligned acc dinp", gu.to_f64(dinp).reshape(N, C), r[0], d, "act_bwd",
              sc["dinp"])
    tol.check("misaligned acc dweight", gu.to_f64(dw), r[1], d, "param_grad", sc["dweight"])
    tol.check("misaligned acc dbias", gu.to_f64(db), r[2], d, "param_grad", sc["dbias"])


def test_accumulate_is_deterministic(lib):
    """Accumulating into the same previous values gives the same bits every
    time (fixed summation order everywhere)."""
    batch = gu.full_batch("gpt2_124m_bf16")
    extras = gu.full_extras("gpt2_124m_bf16")
    w = batch.workload
    inp, wt, bs, dout = gu.batch_to_device(batch)
    out, mean, rstd = gu.forward(lib, inp, wt, bs, w.N, w.C, batch.eps, w.dtype)
    outs = []
    for _ in range(3):
        dinp = gu.to_device(extras.dinp_prev, w.dtype)
        dw = torch.from_numpy(extras.dweight_prev.copy()).cuda()
        db = torch.from_numpy(extras.dbias_prev.copy()).cuda()
        lib.ln_backward_ex(dinp, dw, db, dout, inp, wt, mean, rstd, w.N, w.C, batch.eps,
                           gu.DT[w.dtype], ACC_DINP | ACC_PARAMS)
        outs.append((dinp.view(torch.int16).clone(), dw.clone(), db.clone()))
    for o in outs[1:]:
        assert torch.equal(o[0], outs[0][0])
        assert torch.equal(o[1].view(torch.int32), outs[0][1].view(torch.int32))
        assert torch.equal(o[2].view(torch.int32), outs[0][2].view(torch.int32))
    assert lib.device_status() == 0


def test_variant_edges(lib):
    """N == 0: accumulated parameters are left as they are, overwritten ones
    are zeroed; the recomputing call needs no mean/rstd; unknown flags are
    refused before any launch."""
    C = 64
    dw = torch.full((C,), 3.5, device="cuda")
    db = torch.full((C,), -1.25, device="cuda")
    lib.ln_backward_ex(None, dw, db, None, None, None, None, None, 0, C, 1e-5, 0, ACC_PARAMS)
    torch.cuda.synchronize()
    assert torch.all(dw == 3.5) and torch.all(db == -1.25)
    lib.ln_backward_ex(None, dw, db, None, None, None, None, None, 0, C, 1e-5, 0, RECOMPUTE)
    torch.cuda.synchronize()
    assert torch.all(dw == 0) and torch.all(db == 0)
    n0 = lib.launch_count()
    with pytest.raises(lib.LNError) as e:
        lib.ln_backward_ex(dw, dw, db, dw, dw, dw, None, None, 1, C, 1e-5, 0, 16)
    assert e.value.status == lib.LN_ERR_FLAGS and lib.launch_count() == n0
    # C = 1: every row is constant; recomputed rstd = 1/sqrt(eps), dinp = 0
    x = torch.randn(5, 1, device="cuda")
    dinp = torch.full((5, 1), 7.0, device="cuda")
    lib.ln_backward_ex(dinp, dw[:1], db[:1], torch.ones(5, 1, device="cuda"), x,
                       torch.ones(1, device="cuda"), None, None, 5, 1, 1e-5, 0,
                       ACC_DINP | RECOMPUTE)
    torch.cuda.synchronize()
    assert torch.all(dinp == 7.0), "dinp of a one-column row is zero; 7 + 0 = 7"


def test_fp16_variants_gpt2_124m_shape(lib):
    """fp16 at the GPT-2 124M shape: the residual forward (sum bit-exact) and
    the backward accumulating with recomputed statistics, every element."""
    batch = wl.custom("f16", 65536, 768, seed=20240531, dout_sigma=0.02)
    extras = wl.generate_extras(batch.workload)
    res = _residual(lib, batch, extras, "f16 65536x768")
    res += _backward_ex(lib, batch, extras, FLAG_SETS["acc_recompute"], "f16 65536x768 acc_rec")
    print(res)
