"""B200-native FP4 paged decode attention (BitDecoding-FP4 hot path).

``bdfp4`` is the ctypes binding of the CUDA library ``libbdfp4.so`` (C ABI in
``include/bdfp4.h``); ``workloads`` draws seeded synthetic inputs.
"""
from . import bdfp4, workloads  # noqa: F401
