"""LayerNorm forward and analytical backward for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libln.so`` built from ``csrc/``
(declared in ``include/ln.h``); ``layernorm_fwd_bwd_b200.ln`` is its thin
ctypes binding.  ``layernorm_fwd_bwd_b200.workloads`` draws seeded synthetic
inputs and holds no LayerNorm arithmetic.

The binding is imported lazily so that the input generator can be used on a
machine where the CUDA library has not been built; calling any entry point
without the library raises immediately (there is no CPU fallback).
"""

# Names forwarded to the binding: the entry points (ln_*, raw_*), the
# constants of include/ln.h (LN_*) and the helpers below.  Anything else, the
# submodules included, is not routed through the binding, so importing
# ``workloads`` or ``build`` never needs the built library.
_BINDING_PREFIXES = ("ln_", "LN_", "raw_")
_BINDING_NAMES = ("LNError", "library_path", "launch_count", "version", "device_status",
                  "last_cuda_error", "set_workspace_limit")


def __getattr__(name):
    if name.startswith(_BINDING_PREFIXES) or name in _BINDING_NAMES:
        from . import ln
        try:
            return getattr(ln, name)
        except AttributeError:
            pass
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
