"""ln_backward_noalloc: the backward for callers that cannot allocate device
memory (a fixed arena reserved at start-up, code running inside another
allocator, memory accounting that must not see a second pool).  It keeps its
partial sums in a static device array inside the library instead of the
stream-ordered pool ln_backward uses.

Checked through the C ABI against ln_backward on the same inputs, within the
tolerances the other parity tests use, on two calls in a row: with different
inputs of one shape, and with a second shape on fewer blocks or another row
width (the static array keeps the first call's contents, so the second call
shows that nothing stale leaks in).  This file is collected last so that a run
stopping at its first failure has already run every other test."""
import pytest
import torch

import gpu_util as gu
import tolerances as tol
from layernorm_fwd_bwd_b200 import workloads as wl

pytestmark = pytest.mark.gpu

CASES = [
    ("bf16", 4096, 768),     # one warp per row, grid not limited by the array
    ("bf16", 300, 16384),    # 16 warps per row; the array caps the grid at 32 blocks
    ("f32", 1000, 1600),     # 4 warps per row
    ("f32", 513, 7),         # scalar path
]


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return gu.ln()


def _stats(lib, batch, dev):
    w = batch.workload
    inp, wt, bs, _ = dev
    _, mean, rstd = gu.forward(lib, inp, wt, bs, w.N, w.C, batch.eps, w.dtype)
    return mean, rstd


def _noalloc(lib, dout, inp, wt, mean, rstd, N, C, dtype):
    dinp = gu.nan_tensor((N, C), gu.TORCH_DT[dtype])
    dw = gu.nan_tensor((C,), torch.float32)
    db = gu.nan_tensor((C,), torch.float32)
    lib.ln_backward_noalloc(dinp, dw, db, dout, inp, wt, mean, rstd, N, C, gu.DT[dtype])
    return dinp, dw, db


@pytest.mark.parametrize("dtype,N,C", CASES)
def test_noalloc_matches_ln_backward_twice(lib, dtype, N, C):
    for call, seed in enumerate((101, 202)):
        batch = wl.custom(dtype, N, C, seed=seed + C)
        dev = gu.batch_to_device(batch)
        inp, wt, _, dout = dev
        mean, rstd = _stats(lib, batch, dev)
        want = gu.backward(lib, dout, inp, wt, mean, rstd, N, C, dtype)
        got = _noalloc(lib, dout, inp, wt, mean, rstd, N, C, dtype)
        torch.cuda.synchronize()
        for name, kind, g, r in zip(("dinp", "dweight", "dbias"),
                                    ("act_bwd", "param_grad", "param_grad"), got, want):
            assert not bool(torch.isnan(g.float()).any()), f"call {call}: {name} not written"
            tol.check(f"call {call} {dtype} {N}x{C} {name}", gu.to_f64(g), gu.to_f64(r),
                      dtype, kind)


# Two calls in a row with different shapes, the second on fewer blocks or a
# different row width than the first: the array still holds the first call's
# partial rows (laid out for its C), so a finalise that read a row its own
# call did not write would change dweight or dbias.
SEQUENCES = [
    (("bf16", 300, 16384), ("bf16", 64, 768)),     # 32 capped blocks, then 5 blocks
    (("f32", 1000, 1600), ("bf16", 4096, 768)),
    (("bf16", 4096, 768), ("bf16", 20, 1024)),
    (("f16", 2048, 1600), ("f32", 513, 7)),        # then the scalar path
]


@pytest.mark.parametrize("first,second", SEQUENCES)
def test_noalloc_after_a_different_shape(lib, first, second):
    for call, (dtype, N, C) in enumerate((first, second)):
        batch = wl.custom(dtype, N, C, seed=707 + 13 * call + C)
        dev = gu.batch_to_device(batch)
        inp, wt, _, dout = dev
        mean, rstd = _stats(lib, batch, dev)
        want = gu.backward(lib, dout, inp, wt, mean, rstd, N, C, dtype)
        got = _noalloc(lib, dout, inp, wt, mean, rstd, N, C, dtype)
        torch.cuda.synchronize()
        for name, kind, g, r in zip(("dinp", "dweight", "dbias"),
                                    ("act_bwd", "param_grad", "param_grad"), got, want):
            assert not bool(torch.isnan(g.float()).any()), f"call {call}: {name} not written"
            tol.check(f"call {call} {dtype} {N}x{C} {name}", gu.to_f64(g), gu.to_f64(r),
                      dtype, kind)


def test_noalloc_rejects_wide_rows(lib):
    C = lib.LN_NOALLOC_MAX_C + 1
    before = lib.launch_count()
    with pytest.raises(lib.LNError) as e:
        lib.ln_backward_noalloc(16, 16, 16, 16, 16, 16, 16, 16, 1, C, lib.LN_BF16)
    assert e.value.status == lib.LN_ERR_SCRATCH
    assert "scratch" in lib.ln_status_string(lib.LN_ERR_SCRATCH)
    assert lib.launch_count() == before
