"""Exact online causal long convolution (Flash Inference relaxed schedule) on B200.

The compute path is libfi.so (hand-written CUDA for sm_100a, C-ABI in include/fi.h);
this package only binds it. Import fails loudly if the library has not been built.
"""
from .fi import (Context, FiError, debug_fft, status_str, FI_F32, FI_BF16,  # noqa: F401
                 KERNEL_CLASSES, EXPORTED, LIB_PATH)
