"""B200-native key-gated GLA token mixer of the GTR vision backbone.

The compute lives in ``libgtr_gla.so`` (CUDA C++ for sm_100a, C ABI in
include/gtr_gla.h); :mod:`.gtr_gla` is its ctypes binding (the library is
loaded on first use) and :mod:`.synthetic` draws the seeded synthetic inputs.
"""
from . import synthetic  # noqa: F401
from . import gtr_gla  # noqa: F401

__all__ = ["synthetic", "gtr_gla"]
