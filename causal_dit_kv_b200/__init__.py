"""Sink + rolling-window KV chunk attention for streaming causal DiTs on B200.

The compute path lives in libsdv2 (CUDA, sm_100a) behind the C ABI declared
in include/sdv2.h; :mod:`.binding` forwards to it and :mod:`.stream`
wraps a cache and a motion state with torch-owned device buffers.
"""
from . import binding  # noqa: F401
from .binding import SDV2Error  # noqa: F401
from .stream import KVCache, MotionState  # noqa: F401
