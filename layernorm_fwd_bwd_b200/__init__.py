"""LayerNorm forward and analytical backward for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libln.so`` built from ``csrc/``
(declared in ``include/ln.h``); ``layernorm_fwd_bwd_b200.ln`` is its thin
ctypes binding.  ``layernorm_fwd_bwd_b200.workloads`` draws seeded synthetic
inputs and holds no LayerNorm arithmetic.

The binding is imported lazily so that the input generator can be used on a
machine where the CUDA library has not been built; calling any entry point
without the library raises immediately (there is no CPU fallback).
"""

_BINDING_NAMES = ("ln_forward", "ln_backward", "ln_status_string", "LNError",
                  "LN_F32", "LN_BF16", "library_path", "launch_count")


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import ln
        return getattr(ln, name)
    raise AttributeError(name)
