"""Hybrid Linear Temporal Attention (SWA + DSWA + GLA / gated delta rule) for B200 (sm_100a).

The operator runs in hand-written CUDA kernels behind the C ABI declared in include/kta.h and
exported by ``libkta.so`` (built in-tree from ``csrc/``). ``kta`` is the thin ctypes binding
that marshals torch CUDA tensors into that ABI; ``synth`` holds the seeded input recipe.
Importing this package does not load the CUDA library; importing ``kta`` does, and fails
loudly if it is missing.
"""
__all__ = ["kta", "synth"]
__version__ = "0.1.0"
