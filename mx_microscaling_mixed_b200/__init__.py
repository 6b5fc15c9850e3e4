"""mx_microscaling_mixed_b200 -- mixed-width MXINT quantisation and GEMM for B200.

The compute lives in ``libmxs.so`` (hand-written CUDA for sm_100a behind the C
ABI declared in ``include/mxs.h``).  ``capi`` is a thin ctypes binding with the
same entry-point names; it loads the library on first use and raises if it is
missing.  Importing this package does not touch the GPU.
"""
from . import inputs  # noqa: F401  (seeded synthetic workloads; no method arithmetic)

__all__ = ["inputs", "capi"]


def __getattr__(name):
    if name == "capi":
        from . import capi as _capi
        return _capi
    raise AttributeError(name)
