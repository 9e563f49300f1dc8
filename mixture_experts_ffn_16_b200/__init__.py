"""B200-native (sm_100a) mixture-of-experts FFN block.

The compute path is the C-ABI library ``libmoe.so`` (hand-written CUDA kernels,
declared in ``include/moe.h``); ``api`` is its thin ctypes binding.  Nothing in
this package computes the block on the CPU: calls fail loudly when the CUDA
library is missing.
"""
__all__ = ["api", "inputs"]
