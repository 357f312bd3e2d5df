"""Low-bit recurrent-state decode for B200 (sm_100a).

The computation lives in liblrs.so (CUDA kernels behind the C ABI declared in
include/lrs.h); `lrs` is its Python binding, `inputs` the seeded synthetic
workloads, `shard` the batch partitioning across processes.
"""
from . import lrs  # noqa: F401
