"""B200-native (sm_100a) DeepSeek-V4 hybrid compressed attention core.

The compute lives in libdsv4.so (C ABI declared in include/dsv4.h); ``abi`` binds it
with ctypes and ``harness`` wires workloads onto it.  Importing ``abi`` does not load
the library; the first call does, and fails loudly if it has not been built.
"""
from . import abi  # noqa: F401

__all__ = ["abi"]
