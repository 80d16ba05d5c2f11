"""The seeded input generator (CPU only)."""
import numpy as np
import pytest

from layernorm_fwd_bwd_b200 import workloads as wl


def test_splitmix64_published_values():
    # SplitMix64 with state seed + k*gamma; seed 0 first outputs as published
    # with the algorithm (Steele, Lea, Flood 2014; Vigna's splitmix64.c).
    z = np.uint64(0) + wl.GAMMA
    assert int(wl.raw64(0, 0, np.array([0], np.uint64))[0]) == int(wl._finalise(np.array([z]))[0])
    # seed 0: the first three SplitMix64 outputs
    first = [int(v) for v in wl.raw64(0, 0, np.arange(3, dtype=np.uint64))]
    assert first == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_rows_subset_matches_full():
    work = wl.Workload("t", wl.BF16, 300, 40, 7, dout_sigma=0.02)
    full = wl.generate(work)
    rows = np.array([0, 5, 17, 299])
    part = wl.generate(work, rows)
    assert np.array_equal(full.inp[rows], part.inp)
    assert np.array_equal(full.dout[rows], part.dout)
    assert np.array_equal(full.weight, part.weight)


def test_bf16_rounding_is_nearest_even():
    one = 1.0
    ulp = 2.0 ** -7
    v = np.array([one + ulp / 2, one + 1.5 * ulp, one + ulp / 2 + 1e-12, -3.0,
                  0.0, 1e-3])
    bits = wl.round_bf16_bits(v)
    back = wl.bf16_bits_to_f64(bits)
    assert back[0] == 1.0                 # tie -> even (down)
    assert back[1] == one + 2 * ulp       # tie -> even (up)
    assert back[2] == one + ulp           # above the tie -> up
    assert back[3] == -3.0 and back[4] == 0.0
    assert abs(back[5] - 1e-3) <= 1e-3 * 2.0 ** -8


def test_distributions():
    b = wl.generate(wl.WORKLOADS["gpt2_124m_bf16"], rows=np.arange(512))
    x, dy = b.f64("inp"), b.f64("dout")
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    assert abs(dy.std() - 0.02) < 0.001
    assert abs(b.f64("weight").mean() - 1) < 0.02
    s = wl.generate(wl.WORKLOADS["stress_fp32_65536x768"], rows=np.arange(0, 1000))
    xs = s.f64("inp")
    const = np.arange(1000) % 100 == 0
    assert np.all(xs[const].std(axis=1) == 0)
    assert np.all(np.abs(xs[~const].std(axis=1) - 0.01) < 0.002)
    assert abs(xs.mean() - 100) < 0.01


def test_compulsory_bytes():
    w = wl.WORKLOADS["gpt2_124m_bf16"]
    assert w.fwd_bytes() == 201_853_952
    assert w.bwd_bytes() == 302_521_856
    assert wl.WORKLOADS["stress_fp32_65536x768"].fwd_bytes() + \
        wl.WORKLOADS["stress_fp32_65536x768"].bwd_bytes() == 1_007_696_896


@pytest.mark.parametrize("name,fwd,bwd", [
    ("fp32_256x768", 1_581_056, 2_370_560),
    ("gpt2_124m_bf16", 201_853_952, 302_521_856),
    ("gpt2_350m_bf16", 134_483_968, 201_598_976),
    ("gpt2_1558m_bf16", 104_995_072, 157_433_472),
    ("stress_fp32_65536x768", 403_183_616, 604_513_280),
])
def test_compulsory_bytes_every_workload(name, fwd, bwd):
    """The per-call byte counts every GB/s figure divides by, against the
    table computed independently when the workloads were specified."""
    w = wl.WORKLOADS[name]
    assert (w.fwd_bytes(), w.bwd_bytes()) == (fwd, bwd)


def test_variant_bytes_follow_from_the_plain_calls():
    """Each variant's compulsory bytes differ from the plain call's by exactly
    the arrays it adds or drops: the residual forward reads branch and writes
    resid_out (2NCs more); accumulating reads the previous dinp (NCs) and
    reads dweight/dbias (8C); recomputing reads no saved statistics (8N
    fewer)."""
    import bench
    for w in wl.WORKLOADS.values():
        N, C, s = w.N, w.C, w.elem_bytes
        v = bench.variant_bytes(w)
        assert v["fwd_residual"] == w.fwd_bytes() + 2 * N * C * s
        assert v["bwd_accumulate"] == w.bwd_bytes() + N * C * s + 8 * C
        assert v["bwd_recompute"] == w.bwd_bytes() - 8 * N
        assert v["bwd_accumulate_recompute"] == w.bwd_bytes() + N * C * s + 8 * C - 8 * N


def test_f16_storage_roundtrip():
    """fp16 storage holds numpy's nearest-even float16 of each draw, as 16-bit
    patterns, and reads back exactly."""
    b = wl.custom("f16", 8, 40, seed=9)
    x = b.f64("inp")
    assert b.inp.dtype == np.uint16
    assert np.array_equal(x, b.inp.view(np.float16).astype(np.float64))
    raw = wl._rows_block(b.workload, np.arange(8), wl.S_INP, 0.0, 1.0)
    assert np.array_equal(x, raw.astype(np.float16).astype(np.float64))
