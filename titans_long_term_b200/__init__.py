"""Titans neural long-term memory on B200 (sm_100a): chunk-wise update + retrieve.

The compute runs in ``libtitans_mem.so`` (hand-written CUDA for sm_100a, C ABI in
include/titans_mem.h); :mod:`titans_long_term_b200.mem` is its Python binding and
:mod:`titans_long_term_b200.synth` the seeded synthetic input generator.
"""
from .mem import Memory, TitansError, new_state  # noqa: F401

__all__ = ["Memory", "TitansError", "new_state"]
