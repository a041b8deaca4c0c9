"""B200-native (sm_100a) decode step of a HySparse2 Cross-Decoder hybrid block.

The compute path is libhs2 (CUDA C++, C ABI, ``include/hs2.h``); ``hs2`` is its
ctypes binding and ``workloads`` the seeded synthetic input generator.  Importing
the package loads nothing; the library is loaded on first use.
"""
__all__ = ["hs2", "workloads", "build"]
