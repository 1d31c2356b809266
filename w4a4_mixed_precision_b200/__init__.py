"""Atom W4A4 mixed-precision hot path for B200 (sm_100a).

The compute lives in `libatom_b200.so` (hand-written CUDA, C ABI in
include/atom.h); `atom` is its thin ctypes binding and `inputs` the seeded
synthetic workload generator.
"""
from . import inputs  # noqa: F401

__all__ = ["inputs", "atom"]
