"""B200 (sm_100a) library for the KVSculpt distillation solve.

The work runs in ``libkvsculpt.so`` (CUDA kernels behind the C ABI declared in
``include/kvsculpt.h``).  This package is a thin ctypes binding with the same
entry-point names: it marshals torch tensors (device memory) and CUDA streams
into the C calls and raises on error codes.  There is no fallback path: if the
shared library is missing, importing this package fails.
"""
from ._lib import *  # noqa: F401,F403
from ._lib import __all__  # noqa: F401
