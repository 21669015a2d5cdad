"""B200 (sm_100a) decode step of a very sparse MXFP4 mixture-of-experts layer.

The work is done by the CUDA library libmoe_decode.so (C ABI in
include/moe_decode.h); `api` is its ctypes binding.
"""
from .api import *  # noqa: F401,F403
from .api import EXPORTS, MoEError, load_library  # noqa: F401
