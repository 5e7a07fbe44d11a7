"""FP4 dense attention for long non-causal sequences on NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``libfp4attn.so`` behind the C ABI in
``include/fp4attn.h``; ``nvfp4_precision_b200.fp4attn`` is its ctypes binding
(importing it fails loudly when the library is missing).  ``synth`` holds the
seeded synthetic input generators.
"""
import importlib

__all__ = ["fp4attn", "synth", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
