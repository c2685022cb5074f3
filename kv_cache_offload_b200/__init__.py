"""B200-native zero-copy KV-cache-offload decode step (libdkv) and its Python binding.

The compute lives in libdkv.so (hand-written sm_100a kernels behind the C ABI declared in
include/dkv.h and include/dkv_placement.h); `binding` marshals torch tensors into those
calls.
"""
from .binding import *  # noqa: F401,F403
from .binding import lib, header_symbols, DkvError, BlockManager, read_plan  # noqa: F401
