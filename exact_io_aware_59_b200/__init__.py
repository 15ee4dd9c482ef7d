"""exact_io_aware_59_b200: exact fused attention forward for B200 (sm_100a).

The compute lives in a C-ABI shared library (``libfa_b200.so``, declared in
``include/fa.h``).  ``exact_io_aware_59_b200.binding`` marshals torch tensors into that
ABI; it is loaded lazily so that importing the package (for example to reach
``inputs``) does not need the library.
"""
__all__ = ["binding", "inputs"]
