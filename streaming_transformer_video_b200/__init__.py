"""FlashDecoder streaming step on NVIDIA B200 (sm_100a).

The decoder runs in libflashdec.so (hand-written CUDA for sm_100a behind the
C ABI in include/flashdec.h); this package is its Python binding.
"""
from .flashdec import (FD_BF16, FD_F32, FDError, FlashDecoder, KERNEL_KINDS,  # noqa: F401
                       LIB_PATH, lib, load_library, make_config)
