"""libkvc for NVIDIA B200: a compressed, mixed-format paged KV cache (BF16 /
FP8 e4m3 / packed ternary pages) and single-token decode attention directly
over it.  The compute lives in libkvc.so (CUDA, sm_100a, C ABI in
include/kvc.h); this package is its ctypes binding."""

from .kvc import *  # noqa: F401,F403
from .kvc import (EXPORTS, KvcError, LIB_PATH, kvc_paged_cache,  # noqa: F401
                  make_paged_cache)
from . import paged_cache  # noqa: F401,E402
