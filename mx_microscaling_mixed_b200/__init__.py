"""mx_microscaling_mixed_b200 -- mixed-width MXINT quantisation and GEMM for B200.

The compute lives in ``libmxs.so`` (hand-written CUDA for sm_100a behind the C
ABI declared in ``include/mxs.h``).  ``mx_microscaling_mixed_b200.capi`` is a
thin ctypes binding with the same entry-point names; importing it loads the
library and raises if it is missing.  Importing this package alone does not
touch the GPU.
"""
from . import inputs  # noqa: F401  (seeded synthetic workloads; no method arithmetic)

__all__ = ["inputs"]
