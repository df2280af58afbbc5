"""Cut Cross-Entropy hot path for B200 (sm_100a): fused classifier matmul + loss, forward and backward.

The compute runs in ``libcce.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/cce.h``). ``ops`` is the thin ctypes binding and the
autograd wrapper; importing this package does not load the library, the first
call does, and fails loudly if it is missing.
"""
from .ops import (  # noqa: F401
    CCEError,
    cce_forward,
    cce_backward,
    linear_cross_entropy,
    load_library,
    perplexity,
)

__all__ = ["CCEError", "cce_forward", "cce_backward", "linear_cross_entropy", "load_library", "perplexity"]
