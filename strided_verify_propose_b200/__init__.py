"""B200-native Introspective Strided Decoding (ISD) step.

The product is the C-ABI library ``libisd.so`` (declared in include/isd.h)
built from the sm_100a CUDA kernels under ``csrc/``; ``binding`` is its thin
ctypes binding. Importing this package does not load the library; the first
binding call does, and raises if it has not been built.
"""
from . import binding  # noqa: F401

__all__ = ["binding"]
