"""nslm: a B200-native library for SeedLM seed-decompress matrix multiplies.

Expert weights are stored as packed SeedLM blocks (a 16-bit LFSR seed, P int4
coefficients and a 4-bit exponent code per 8 weights) and rebuilt inside the
CUDA kernels of ``libnslm.so``.  ``lfsr_seeded_moe_b200.nslm`` is the thin
ctypes binding to that library; ``lfsr_seeded_moe_b200.synth`` draws seeded
synthetic inputs.  Submodules are imported on first use so the input
generator works on a machine without a GPU.
"""
import importlib

__all__ = ["nslm", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
