"""B200-native denoising step for block-diffusion decoding (Fast-dLLM / v2).

The compute lives in ``libfdl.so`` (hand-written CUDA for sm_100a behind a
C ABI, declared in ``include/fdl.h``); ``fdl`` is the thin ctypes binding with
the same entry-point names.  ``synth`` draws the seeded synthetic inputs.
Importing the package loads nothing; ``fdl`` loads the library on first use
and raises if it is missing.
"""
__all__ = ["fdl", "synth"]
