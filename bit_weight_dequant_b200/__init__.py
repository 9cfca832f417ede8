"""B200-native blockwise 4-bit weight dequantization + fused skinny GEMM.

The compute lives in ``libq4.so`` (hand-written CUDA for sm_100a, C ABI in
``include/q4.h``); this package is its ctypes binding plus the seeded input
generators (``inputs``).  Importing the package does not load the library;
the first call does, and raises if the library has not been built.
"""
from .binding import (Q4Error, Workspace, q4_dequantize_blockwise, q4_gemm_plan, q4_gemm_skinny,  # noqa: F401
                      q4_gemm_workspace_size, q4_quantize_blockwise, status_string)
