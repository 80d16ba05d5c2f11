"""Python binding of libln.so (declared in include/ln.h).

Argument marshalling only: every array argument may be a CUDA ``torch.Tensor``
(its ``data_ptr()`` is passed), a plain integer device address, or ``None``
(NULL).  ``stream`` may be a ``torch.cuda.Stream``, a raw ``cudaStream_t``
integer, or ``None`` for PyTorch's current stream on the current device.
The caller owns all memory and must make the right device current.

All computation happens in the CUDA library.  If ``libln.so`` has not been
built, importing this module raises ``ImportError``; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libln.so")

LN_F32 = 0
LN_BF16 = 1
LN_F16 = 2

LN_OK = 0
LN_ERR_NULL = 1
LN_ERR_SHAPE = 2
LN_ERR_DTYPE = 3
LN_ERR_EPS = 4
LN_ERR_WORKSPACE = 5
LN_ERR_CUDA = 6
LN_ERR_SCRATCH = 7
LN_ERR_FLAGS = 8
LN_ERR_ALIAS = 9
LN_BWD_ACCUMULATE_DINP = 1
LN_BWD_ACCUMULATE_DPARAMS = 2
LN_BWD_RECOMPUTE_STATS = 4
LN_NOALLOC_SCRATCH_BYTES = 4 << 20
LN_NOALLOC_MAX_C = LN_NOALLOC_SCRATCH_BYTES // 8
LN_MAX_C = 1 << 24
LN_MAX_N = 1 << 40
LN_MAX_ELEMS = 1 << 50

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with "
        "`python -m layernorm_fwd_bwd_b200.build` (nvcc, sm_100a)")

_lib = ctypes.CDLL(_LIB_PATH)
_vp, _i64, _int, _f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
_lib.ln_forward.restype = _int
_lib.ln_forward.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _f32, _int, _vp]
_lib.ln_backward.restype = _int
_lib.ln_backward.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _int, _vp]
_lib.ln_backward_noalloc.restype = _int
_lib.ln_backward_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64,
                                     _int, _vp]
_lib.ln_forward_residual.restype = _int
_lib.ln_forward_residual.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _f32,
                                     _int, _vp]
_lib.ln_backward_ex.restype = _int
_lib.ln_backward_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _f32, _int,
                                ctypes.c_uint, _vp]
_lib.ln_status_string.restype = ctypes.c_char_p
_lib.ln_status_string.argtypes = [_int]
_lib.ln_launch_count.restype = ctypes.c_uint64
_lib.ln_launch_count.argtypes = []
_lib.ln_version.restype = _int
_lib.ln_version.argtypes = []
_lib.ln_device_status.restype = _int
_lib.ln_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint), _int]
_lib.ln_set_workspace_limit.restype = _int
_lib.ln_set_workspace_limit.argtypes = [_i64]
_lib.ln_last_cuda_error.restype = ctypes.c_char_p
_lib.ln_last_cuda_error.argtypes = []


class LNError(RuntimeError):
    """A non-LN_OK status; for LN_ERR_CUDA the message also names the CUDA
    error and the runtime call that raised it."""

    def __init__(self, status: int):
        self.status = status
        msg = ln_status_string(status)
        if status == LN_ERR_CUDA:
            msg += f" [{last_cuda_error()}]"
        super().__init__(msg)


def library_path() -> str:
    return _LIB_PATH


def ln_status_string(status: int) -> str:
    return _lib.ln_status_string(int(status)).decode()


def launch_count() -> int:
    return int(_lib.ln_launch_count())


def version() -> int:
    return int(_lib.ln_version())


def last_cuda_error() -> str:
    """The CUDA error behind this thread's most recent LN_ERR_CUDA."""
    return _lib.ln_last_cuda_error().decode()


def set_workspace_limit(nbytes: int) -> None:
    """Cap the pooled backward's workspace per call on the current device
    (0: no cap); a call needing more fails with LN_ERR_WORKSPACE."""
    _check(_lib.ln_set_workspace_limit(int(nbytes)))


def device_status(clear: bool = False) -> int:
    """Bits set on the current device by kernels whose bounded waits ran out
    (0: healthy).  Synchronises the device."""
    bits = ctypes.c_uint(0)
    _check(_lib.ln_device_status(ctypes.byref(bits), int(bool(clear))))
    return int(bits.value)


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc: int) -> None:
    if rc != LN_OK:
        raise LNError(rc)


def ln_forward(out, mean, rstd, inp, weight, bias, N: int, C: int, eps: float,
               dtype: int, stream=None) -> None:
    """out, mean, rstd <- LayerNorm(inp; weight, bias, eps) over N rows of C."""
    _check(_lib.ln_forward(_ptr(out), _ptr(mean), _ptr(rstd), _ptr(inp),
                           _ptr(weight), _ptr(bias), int(N), int(C), float(eps),
                           int(dtype), _stream(stream)))


def ln_backward(dinp, dweight, dbias, dout, inp, weight, mean, rstd, N: int,
                C: int, dtype: int, stream=None) -> None:
    """dinp, dweight, dbias <- analytical LayerNorm backward of dout."""
    _check(_lib.ln_backward(_ptr(dinp), _ptr(dweight), _ptr(dbias), _ptr(dout),
                            _ptr(inp), _ptr(weight), _ptr(mean), _ptr(rstd),
                            int(N), int(C), int(dtype), _stream(stream)))


def ln_forward_residual(resid_out, out, mean, rstd, resid, branch, weight, bias, N: int,
                        C: int, eps: float, dtype: int, stream=None) -> None:
    """resid_out <- resid + branch (rounded to dtype); out, mean, rstd <-
    LayerNorm(resid_out; weight, bias, eps).  No output may overlap another
    output or an input (LN_ERR_ALIAS)."""
    _check(_lib.ln_forward_residual(_ptr(resid_out), _ptr(out), _ptr(mean), _ptr(rstd),
                                    _ptr(resid), _ptr(branch), _ptr(weight), _ptr(bias),
                                    int(N), int(C), float(eps), int(dtype), _stream(stream)))


def ln_backward_ex(dinp, dweight, dbias, dout, inp, weight, mean, rstd, N: int, C: int,
                   eps: float, dtype: int, flags: int, stream=None) -> None:
    """ln_backward with variants selected by ``flags`` (LN_BWD_ACCUMULATE_DINP:
    dinp +=; LN_BWD_ACCUMULATE_DPARAMS: dweight/dbias +=;
    LN_BWD_RECOMPUTE_STATS: mean/rstd recomputed from inp with eps, so they
    may be None)."""
    _check(_lib.ln_backward_ex(_ptr(dinp), _ptr(dweight), _ptr(dbias), _ptr(dout),
                               _ptr(inp), _ptr(weight), _ptr(mean), _ptr(rstd), int(N),
                               int(C), float(eps), int(dtype), int(flags), _stream(stream)))


def ln_backward_noalloc(dinp, dweight, dbias, dout, inp, weight, mean, rstd, N: int,
                        C: int, dtype: int, stream=None) -> None:
    """ln_backward for callers that cannot allocate device memory: its partial
    sums live in a static device array inside the library (4 MiB per GPU),
    so C is limited to LN_NOALLOC_MAX_C and calls that overlap on the GPU
    race on that array; the first call on a device must precede any stream
    capture."""
    _check(_lib.ln_backward_noalloc(_ptr(dinp), _ptr(dweight), _ptr(dbias), _ptr(dout),
                                    _ptr(inp), _ptr(weight), _ptr(mean), _ptr(rstd),
                                    int(N), int(C), int(dtype), _stream(stream)))


def raw_forward(*args) -> int:
    """Call ln_forward with already-marshalled arguments; returns the status."""
    return int(_lib.ln_forward(*args))


def raw_backward(*args) -> int:
    """Call ln_backward with already-marshalled arguments; returns the status."""
    return int(_lib.ln_backward(*args))


def raw_forward_residual(*args) -> int:
    """Call ln_forward_residual with already-marshalled arguments; returns the
    status."""
    return int(_lib.ln_forward_residual(*args))


def raw_backward_ex(*args) -> int:
    """Call ln_backward_ex with already-marshalled arguments; returns the status."""
    return int(_lib.ln_backward_ex(*args))
