"""FP8 linear layer with per-tensor delayed scaling, for NVIDIA B200 (sm_100a).

The compute lives in ``libfp8dsa.so`` (hand-written CUDA: amax-fused E4M3/E5M2 quantize
with an in-kernel history-ring fold, and a TMA + tcgen05 FP8 GEMM with a fused
dequantize/bias epilogue).  This package is its thin ctypes binding; see
``include/fp8dsa.h`` for the C ABI.
"""

from ._capi import *  # noqa: F401,F403
from ._capi import Ring, FP8Error, lib, header_functions, last_error  # noqa: F401

__all__ = [n for n in dir() if not n.startswith("_")]
