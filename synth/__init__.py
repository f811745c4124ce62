"""Seeded synthetic inputs for the compressed-KV decode path.

This module holds only workload shapes and random draws: no codec, rotary, compressor, scoring,
selection or attention arithmetic. The CUDA path and the CPU oracle both consume the bytes it
produces, each decoding them with its own code.
"""

from .workloads import *  # noqa: F401,F403
