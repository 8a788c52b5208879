"""B200-native group-wise affine quantized matmul (libqmm).

The compute lives in ``libqmm.so`` (hand-written CUDA for sm_100a behind a
C ABI declared in ``include/qmm.h``); ``binding`` marshals torch tensors to
that ABI.  Importing this package does not load the library: the first call
into ``binding`` does, and raises if the library is missing.
"""
__all__ = ["binding", "workloads"]
