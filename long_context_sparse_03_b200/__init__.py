"""B200-native CSA / HCA hot path: ctypes binding of libcsa.so.

The compute path is entirely in libcsa.so (hand-written CUDA for sm_100a,
C ABI declared in include/csa.h); this package only marshals torch device
tensors into that ABI.  There is no CPU fallback: importing the binding
without the built library raises.
"""
from .workloads import Workload  # noqa: F401

__all__ = ["Workload"]
