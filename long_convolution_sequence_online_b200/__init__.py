"""Exact online causal long convolution (Flash Inference relaxed schedule) on B200.

The compute path is libfi.so (hand-written CUDA for sm_100a, C-ABI in include/fi.h);
this package only binds it. The binding (module `fi`) loads the library on first use
and raises if it has not been built: there is no fallback path.
"""
_EXPORTS = ("Context", "FiError", "debug_fft", "status_str", "FI_F32", "FI_BF16", "KERNEL_CLASSES",
            "EXPORTED", "LIB_PATH")


def __getattr__(name):
    if name in _EXPORTS:
        from . import fi
        return getattr(fi, name)
    raise AttributeError(name)
