"""B200-native (sm_100a) exact tiled attention.

The product is the C-ABI library ``libfa_b200.so`` (declared in
``include/fa.h``); :mod:`exact_io_aware_63_b200.binding` is its thin ctypes
binding and :mod:`exact_io_aware_63_b200.inputs` draws the seeded synthetic
workloads.  Importing this package loads nothing; the library is loaded on
first use and its absence is an error (there is no CPU fallback).
"""

__all__ = ["binding", "build", "inputs"]
