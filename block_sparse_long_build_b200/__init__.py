"""Block-sparse long-context attention for B200 (sm_100a).

The computation lives in libbsa.so (CUDA kernels behind a C ABI declared in
include/bsa.h).  ``native`` is its ctypes binding, ``session`` sequences the
calls of a decode step, ``workloads`` draws seeded synthetic inputs.
"""
from . import native, workloads  # noqa: F401

__all__ = ["native", "workloads"]
