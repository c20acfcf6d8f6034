"""Lossless BF16 exponent compression (Unweight-style) with B200 kernels.

The compute path is the C-ABI library ``libuw.so`` built from ``csrc/``;
``uw`` is its thin ctypes binding.  ``synth`` generates seeded inputs.
Nothing is imported eagerly, so ``synth`` can be used without the library.
"""
__all__ = ["uw", "synth"]
