"""RIPE verify attention for looped language models on B200 (sm_100a).

The CUDA library (``lib/libripe.so``, C ABI in ``include/ripe.h``) holds the
hot path; ``ripe`` is its Python binding and ``synth`` draws seeded synthetic
inputs.
"""
__all__ = ["ripe", "synth", "build"]
