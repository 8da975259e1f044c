"""LeapQuant int8-state GDN/KDA decode step for B200 (sm_100a).

The compute lives in the C-ABI library libleapquant.so (CUDA kernels for
sm_100a, declared in include/leapquant.h).  `binding` is its thin ctypes
binding; it raises at import time if the library has not been built.
`workloads` draws the seeded synthetic inputs.
"""
__all__ = ["binding", "workloads"]
