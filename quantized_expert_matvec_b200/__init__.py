"""B200-native quantized MoE expert step (sm_100a CUDA kernels behind a C ABI).

The compute runs in ``libqexpert.so`` (see ``include/qexpert.h``); this
package is a thin ctypes binding that marshals torch CUDA tensors to the C
entry points.  There is no CPU fallback: importing the binding raises if the
shared library is missing.
"""
from ._binding import *  # noqa: F401,F403
from ._binding import __all__  # noqa: F401
