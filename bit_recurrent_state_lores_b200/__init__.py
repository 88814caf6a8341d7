"""LoReS quantized recurrent-state decode step for B200 (sm_100a).

The product is the C-ABI library liblores.so (include/lores.h); this package holds
its CUDA sources (csrc/), the build step (build.py), the ctypes binding (lores.py)
and seeded synthetic workloads (synth.py).  The binding's names are re-exported
here on first use; that import fails loudly when the library has not been built:
there is no CPU fallback.
"""
import importlib


# submodules: `from bit_recurrent_state_lores_b200 import synth` must not load the library
_SUBMODULES = ("synth", "build", "lores")


def __getattr__(name):
    if name.startswith("__") or name in _SUBMODULES:
        raise AttributeError(name)
    mod = importlib.import_module(__name__ + ".lores")
    try:
        return getattr(mod, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None
