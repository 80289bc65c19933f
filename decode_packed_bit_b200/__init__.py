"""decode_packed_bit_b200: packed low-bit GEMV/GEMM kernels for NVIDIA B200.

The compute lives in liblowbit.so (hand-written CUDA for sm_100a, C ABI in
include/lowbit.h); ``decode_packed_bit_b200.lowbit`` is its Python binding.
"""
from .lowbit import *  # noqa: F401,F403
from .lowbit import LowbitError, lib  # noqa: F401
