"""SmoothQuant W8A8 linear-layer path and LLM.int8() decomposition for B200.

The compute lives in libsq_b200.so (hand-written CUDA for sm_100a behind a C
ABI, declared in include/sq_api.h); ``_lib`` is its ctypes binding. Import of
this package does not load the library; the first call does, and raises if
the library is missing. ``inputs`` holds the seeded synthetic workloads.
"""
from . import _lib  # noqa: F401
from ._lib import *  # noqa: F401,F403
