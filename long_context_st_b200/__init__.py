"""JoLT KV-cache codec for NVIDIA B200: C ABI (include/jolt.h) + hand-written sm_100a kernels.

Python side: `long_context_st_b200.api` (ctypes marshalling only) and `build` (in-tree nvcc).
"""
from . import api  # noqa: F401
from ._lib import lib, LIB_PATH, JoltError  # noqa: F401
