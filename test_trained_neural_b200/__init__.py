"""B200-native (sm_100a) chunked write-and-read of the Titans neural memory.

The compute lives in libtitansmem.so (CUDA, C ABI in include/titansmem.h);
this package is its thin Python binding.
"""
from .memory import NeuralMemory, prologue  # noqa: F401
from ._native import TitansMemError  # noqa: F401
