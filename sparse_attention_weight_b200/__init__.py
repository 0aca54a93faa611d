"""B200-native DeepSeek Sparse Attention (DSA) hot path.

The compute lives in ``libdsa.so`` (hand-written CUDA for sm_100a behind a
C ABI, declared in include/dsa.h).  ``binding`` marshals torch tensors into
that ABI; importing this package does not load the library.
"""
from .configs import WORKLOADS, Workload  # noqa: F401
