"""kvattn: single-token decode attention over a KV cache on NVIDIA B200 (sm_100a).

The compute lives in the C-ABI shared library ``libkvattn.so`` (CUDA kernels for
sm_100a, declared in ``include/kvattn.h``).  This package holds that library's
sources (``csrc/``), its build step (``build.py``), a thin ctypes binding with the
same names as the C entry points (``binding.py``) and the seeded synthetic inputs
(``workloads.py``).  Importing the package loads nothing; the first call into the
binding loads the library and raises if it is missing.  There is no CPU fallback.
"""

__all__ = ["binding", "workloads", "build"]
