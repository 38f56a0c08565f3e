"""B200-native (sm_100a) quantized self-attention for video diffusion transformers.

The native library ``libsage.so`` (CUDA, C ABI in ``include/sage.h``) holds
the whole path: the quantization prepass (K smoothing, per-block INT8 Q/K,
per-channel FP8 V), the INT8/FP8 tcgen05 attention kernel, the BF16 tcgen05
attention kernel and the per-layer mode table.  ``sage`` is its ctypes
binding.
"""
from . import build  # noqa: F401

__all__ = ["build", "sage"]
