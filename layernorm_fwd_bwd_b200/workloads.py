"""Seeded synthetic LayerNorm workloads.

This module only draws inputs.  It holds none of LayerNorm's arithmetic, so the
CPU oracle and the CUDA path can both take their inputs from it without sharing
any computation.

Generator.  Every element is drawn from a counter-based SplitMix64 stream
(G. Steele, D. Lea, C. Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014): the k-th state of stream ``s`` under seed ``seed`` is
``seed + (s * 2**48 + k + 1) * 0x9E3779B97F4A7C15 (mod 2**64)`` and the draw is
the SplitMix64 finaliser of that state.  Because a draw depends only on its
counter, any subset of rows can be generated on its own and matches the same
rows of the full array.  Normals use the Box-Muller transform (Box & Muller,
1958) on 53-bit uniforms: draws 2p and 2p+1 of a stream give
u1 = (hi53 + 1) / 2**53 in (0, 1] and u2 = hi53 / 2**53 in [0, 1), and the
normals of pair p are r cos(2 pi u2) (even index) and r sin(2 pi u2) (odd
index) with r = sqrt(-2 ln u1).  Values are computed in double and rounded
once, to nearest-even, to the activation dtype.

Workloads.  The five workloads are the shapes GPT-2 training runs LayerNorm on
(rows N = batch * sequence, channels C), plus a small fp32 case and an fp32
cancellation stress case:

=====================  =====  ======  =====  =====================================
name                   dtype  N       C      inp / dout
=====================  =====  ======  =====  =====================================
fp32_256x768           f32    256     768    N(0,1) / N(0,1)
gpt2_124m_bf16         bf16   65536   768    N(0,1) / N(0, 0.02^2)
gpt2_350m_bf16         bf16   32768   1024   N(0,1) / N(0, 0.02^2)
gpt2_1558m_bf16        bf16   16384   1600   N(0,1) / N(0, 0.02^2)
stress_fp32_65536x768  f32    65536   768    100 + 0.01 N(0,1), every 100th row
                                             constant / N(0,1)
=====================  =====  ======  =====  =====================================

weight ~ 1 + 0.1 N(0,1) and bias ~ 0.1 N(0,1) everywhere; eps = 1e-5.  In the
stress case every row r with r % 100 == 0 holds one value v_r = 100 + 0.01 z_r
(one draw per row) in all C columns, so its variance is exactly zero.

Inputs of the variants (``generate_extras``, streams of their own so the
arrays above do not change): the residual branch added to inp by the fused
residual forward, branch ~ N(0, inp_sigma^2) (a sub-layer output at the
residual stream's own spread; in the stress case the sum stays near 100), a
previous dinp for the accumulating backward, N(0, (dout_sigma /
inp_sigma)^2) (the scale of dinp itself, rstd * dout * weight), and previous
dweight and dbias, fp32 N(0,1).
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# stream ids: one per drawn array
S_INP, S_WEIGHT, S_BIAS, S_DOUT, S_CONST = 0, 1, 2, 3, 4
S_BRANCH, S_DINP_PREV, S_PARAM_PREV = 5, 6, 7

EPS = float(np.float32(1e-5))

F32, BF16, F16 = "f32", "bf16", "f16"


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str           # "f32", "bf16" or "f16": dtype of inp/out/dout/dinp/weight/bias
    N: int               # rows (batch * sequence)
    C: int               # channels
    seed: int
    inp_mu: float = 0.0
    inp_sigma: float = 1.0
    dout_sigma: float = 1.0
    const_row_period: int = 0   # rows r with r % period == 0 are constant (0: none)
    description: str = ""

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == F32 else 2

    def fwd_bytes(self) -> int:
        """Compulsory HBM bytes of one forward pass: read inp, write out,
        write mean and rstd, read weight and bias."""
        s = self.elem_bytes
        return 2 * self.N * self.C * s + 8 * self.N + 2 * self.C * s

    def bwd_bytes(self) -> int:
        """Compulsory HBM bytes of one backward pass: read dout and inp, write
        dinp, read mean and rstd, read weight, write dweight and dbias."""
        s = self.elem_bytes
        return 3 * self.N * self.C * s + 8 * self.N + self.C * s + 8 * self.C


WORKLOADS = {
    w.name: w for w in [
        Workload("fp32_256x768", F32, 256, 768, 20240521,
                 description="fp32, B=4 T=64 (N=256), C=768"),
        Workload("gpt2_124m_bf16", BF16, 65536, 768, 20240522, dout_sigma=0.02,
                 description="GPT-2 124M LayerNorm: bf16, B=64 T=1024 (N=65536), C=768"),
        Workload("gpt2_350m_bf16", BF16, 32768, 1024, 20240523, dout_sigma=0.02,
                 description="GPT-2 350M LayerNorm: bf16, B=32 T=1024 (N=32768), C=1024"),
        Workload("gpt2_1558m_bf16", BF16, 16384, 1600, 20240524, dout_sigma=0.02,
                 description="GPT-2 1.5B LayerNorm: bf16, B=16 T=1024 (N=16384), C=1600"),
        Workload("stress_fp32_65536x768", F32, 65536, 768, 20240525,
                 inp_mu=100.0, inp_sigma=0.01, const_row_period=100,
                 description="fp32 cancellation stress: inp = 100 + 0.01 N(0,1), "
                             "every 100th row constant, N=65536, C=768"),
    ]
}

HEADLINE = "gpt2_124m_bf16"


def _finalise(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def raw64(seed: int, stream: int, counters: np.ndarray) -> np.ndarray:
    """SplitMix64 draws at the given counters of ``stream``."""
    base = np.uint64((seed + (stream << 48) + 1) % (1 << 64))
    with np.errstate(over="ignore"):
        state = (base + counters.astype(np.uint64)) * GAMMA
        return _finalise(state)


def normals(seed: int, stream: int, index: np.ndarray) -> np.ndarray:
    """Standard normals (float64) at element indices ``index`` of ``stream``."""
    index = np.asarray(index, dtype=np.uint64)
    pair = index >> np.uint64(1)
    z1 = raw64(seed, stream, pair << np.uint64(1))
    z2 = raw64(seed, stream, (pair << np.uint64(1)) + np.uint64(1))
    u1 = ((z1 >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53
    u2 = (z2 >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    r = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * math.pi * u2
    odd = (index & np.uint64(1)).astype(bool)
    return np.where(odd, r * np.sin(ang), r * np.cos(ang))


def round_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round float64 values once, to nearest-even, to bfloat16 (8 significant
    bits) and return the 16-bit patterns.  Normal-range values only."""
    m, e = np.frexp(np.asarray(v, dtype=np.float64))
    q = np.ldexp(np.rint(m * 256.0) / 256.0, e)          # exact in bf16
    return (q.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def to_storage(v: np.ndarray, dtype: str) -> np.ndarray:
    """float64 -> storage array (float32, or uint16 bit patterns of bf16 /
    fp16; numpy's float16 cast rounds to nearest-even)."""
    if dtype == F32:
        return np.asarray(v, dtype=np.float64).astype(np.float32)
    if dtype == F16:
        return np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)
    return round_bf16_bits(v)


def storage_to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 values of a storage array."""
    if dtype == F32:
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    if dtype == F16:
        return np.asarray(a, dtype=np.uint16).view(np.float16).astype(np.float64)
    return bf16_bits_to_f64(np.asarray(a, dtype=np.uint16))


@dataclasses.dataclass
class Batch:
    """One batch of inputs in storage form (float32, or uint16 bf16 / fp16
    bits)."""
    workload: Workload
    rows: np.ndarray          # int64 row indices of the workload held here
    inp: np.ndarray           # [len(rows), C]
    weight: np.ndarray        # [C]
    bias: np.ndarray          # [C]
    dout: np.ndarray          # [len(rows), C]
    eps: float = EPS

    def f64(self, name: str) -> np.ndarray:
        return storage_to_f64(getattr(self, name), self.workload.dtype)


def _rows_block(w: Workload, rows: np.ndarray, stream: int, mu: float,
                sigma: float) -> np.ndarray:
    C = w.C
    idx = (rows.astype(np.uint64)[:, None] * np.uint64(C)
           + np.arange(C, dtype=np.uint64)[None, :])
    return mu + sigma * normals(w.seed, stream, idx.reshape(-1)).reshape(len(rows), C)


def generate(w: Workload, rows=None, chunk_rows: int = 8192, workers: int = 0) -> Batch:
    """Draw the workload's inputs for ``rows`` (all rows when None).  Chunks
    of rows are drawn on ``workers`` threads (0: up to 8, by the host's core
    count); the counter-based generator makes every element independent of
    the chunking and of the thread that draws it."""
    rows = np.arange(w.N, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    if rows.size and (rows.min() < 0 or rows.max() >= w.N):
        raise ValueError("row index out of range")
    cidx = np.arange(w.C, dtype=np.uint64)
    weight = to_storage(1.0 + 0.1 * normals(w.seed, S_WEIGHT, cidx), w.dtype)
    bias = to_storage(0.1 * normals(w.seed, S_BIAS, cidx), w.dtype)
    store = np.float32 if w.dtype == F32 else np.uint16
    inp = np.empty((rows.size, w.C), store)
    dout = np.empty((rows.size, w.C), store)

    def chunk(a):
        rr = rows[a:a + chunk_rows]
        x = _rows_block(w, rr, S_INP, w.inp_mu, w.inp_sigma)
        if w.const_row_period:
            const = rr % w.const_row_period == 0
            if const.any():
                z = normals(w.seed, S_CONST, rr[const].astype(np.uint64))
                x[const, :] = (w.inp_mu + w.inp_sigma * z)[:, None]
        inp[a:a + rr.size] = to_storage(x, w.dtype)
        dout[a:a + rr.size] = to_storage(
            _rows_block(w, rr, S_DOUT, 0.0, w.dout_sigma), w.dtype)

    starts = range(0, rows.size, chunk_rows)
    n = workers or min(8, os.cpu_count() or 1)
    if n > 1 and len(starts) > 1:
        with concurrent.futures.ThreadPoolExecutor(n) as ex:
            list(ex.map(chunk, starts))
    else:
        for a in starts:
            chunk(a)
    return Batch(w, rows, inp, weight, bias, dout)


def custom(dtype: str, N: int, C: int, seed: int, inp_mu: float = 0.0,
           inp_sigma: float = 1.0, dout_sigma: float = 1.0,
           const_row_period: int = 0) -> Batch:
    """A batch of an arbitrary shape drawn the same way (shape sweeps)."""
    w = Workload(f"custom_{dtype}_{N}x{C}", dtype, N, C, seed, inp_mu, inp_sigma,
                 dout_sigma, const_row_period)
    return generate(w)


@dataclasses.dataclass
class Extras:
    """Inputs of the variants, for the same rows as a Batch."""
    workload: Workload
    rows: np.ndarray
    branch: np.ndarray        # [len(rows), C] storage: added to inp (residual forward)
    dinp_prev: np.ndarray     # [len(rows), C] storage: accumulated into (backward)
    dweight_prev: np.ndarray  # [C] float32
    dbias_prev: np.ndarray    # [C] float32

    def f64(self, name: str) -> np.ndarray:
        a = getattr(self, name)
        if name in ("dweight_prev", "dbias_prev"):
            return a.astype(np.float64)
        return storage_to_f64(a, self.workload.dtype)


def generate_extras(w: Workload, rows=None, chunk_rows: int = 8192) -> Extras:
    """Draw the variants' inputs for ``rows`` (all rows when None)."""
    rows = np.arange(w.N, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    if rows.size and (rows.min() < 0 or rows.max() >= w.N):
        raise ValueError("row index out of range")
    store = np.float32 if w.dtype == F32 else np.uint16
    branch = np.empty((rows.size, w.C), store)
    prev = np.empty((rows.size, w.C), store)
    for a in range(0, rows.size, chunk_rows):
        rr = rows[a:a + chunk_rows]
        branch[a:a + rr.size] = to_storage(_rows_block(w, rr, S_BRANCH, 0.0, w.inp_sigma), w.dtype)
        prev[a:a + rr.size] = to_storage(
            _rows_block(w, rr, S_DINP_PREV, 0.0, w.dout_sigma / w.inp_sigma), w.dtype)
    cidx = np.arange(2 * w.C, dtype=np.uint64)
    params = normals(w.seed, S_PARAM_PREV, cidx).astype(np.float32)
    return Extras(w, rows, branch, prev, params[:w.C].copy(), params[w.C:].copy())
