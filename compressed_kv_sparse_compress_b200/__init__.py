"""Compressed-KV sparse decode attention for NVIDIA B200 (sm_100a).

The CUDA library libckv.so (C ABI in include/ckv.h) holds every kernel; this package is its
ctypes binding plus a small decode-step runner. PyTorch supplies device memory and streams.
"""

from .binding import *  # noqa: F401,F403
from .binding import load_library, launch_count, status_str  # noqa: F401
from .decode import DecodeLayer, cache_from_tensors  # noqa: F401
