"""Device-side helpers shared by the GPU tests: move seeded storage arrays to
the GPU, call the C ABI through the binding, and bring results back as
float64.  No LayerNorm arithmetic here."""
from __future__ import annotations

import functools

import numpy as np
import torch

from layernorm_fwd_bwd_b200 import workloads as wl

DT = {"f32": 0, "bf16": 1, "f16": 2}
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def ln():
    from layernorm_fwd_bwd_b200 import build
    build.build()
    from layernorm_fwd_bwd_b200 import ln as binding
    return binding


def to_device(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)
    bits = np.ascontiguousarray(a, np.uint16).view(np.int16)
    return torch.from_numpy(bits).to(device).view(TORCH_DT[dtype])


def to_f64(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return wl.bf16_bits_to_f64(t.view(torch.int16).numpy().view(np.uint16))
    if t.dtype == torch.float16:
        return wl.storage_to_f64(t.view(torch.int16).numpy().view(np.uint16), "f16")
    return t.numpy().astype(np.float64)


def bits(t: torch.Tensor) -> torch.Tensor:
    """The tensor's bit patterns as integers (for bitwise comparisons)."""
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


def nan_tensor(shape, tdtype, device="cuda") -> torch.Tensor:
    return torch.full(shape, float("nan"), dtype=tdtype, device=device)


def forward_outputs(N, C, dtype):
    """NaN-filled out, mean, rstd (so an element the library skips shows)."""
    return (nan_tensor((N, C), TORCH_DT[dtype]), nan_tensor((N,), torch.float32),
            nan_tensor((N,), torch.float32))


def forward(lib, inp, w, b, N, C, eps, dtype, stream=None):
    out = nan_tensor((N, C), TORCH_DT[dtype])
    mean = nan_tensor((N,), torch.float32)
    rstd = nan_tensor((N,), torch.float32)
    lib.ln_forward(out, mean, rstd, inp, w, b, N, C, eps, DT[dtype], stream)
    return out, mean, rstd


def backward(lib, dout, inp, w, mean, rstd, N, C, dtype, stream=None):
    dinp = nan_tensor((N, C), TORCH_DT[dtype])
    dw = nan_tensor((C,), torch.float32)
    db = nan_tensor((C,), torch.float32)
    lib.ln_backward(dinp, dw, db, dout, inp, w, mean, rstd, N, C, DT[dtype], stream)
    return dinp, dw, db


def batch_to_device(batch: wl.Batch):
    d = batch.workload.dtype
    return (to_device(batch.inp, d), to_device(batch.weight, d),
            to_device(batch.bias, d), to_device(batch.dout, d))


@functools.lru_cache(maxsize=2)
def full_batch(name: str) -> wl.Batch:
    """The named workload at its full size (cached: drawing 50M elements takes
    seconds)."""
    return wl.generate(wl.WORKLOADS[name])


@functools.lru_cache(maxsize=2)
def full_extras(name: str) -> wl.Extras:
    """The variants' extra inputs for the named workload at full size."""
    return wl.generate_extras(wl.WORKLOADS[name])
