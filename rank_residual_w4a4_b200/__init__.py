"""B200-native (sm_100a) fused dual-component W4A4 + low-rank linear layer.

Implements the inference hot path of TwinQuant ("TwinQuant: Learnable Subspace
Decomposition for 4-Bit LLM Quantization", §4.3): Y = Q(X)Q(R) +
bf16(Q(X)Q(L1)) L2 with symmetric 4-bit codes (Eq. (1)), per-group-128 fp32
scales, the low-rank intermediate kept on chip and a single epilogue.

The compute lives in libtwq.so (C ABI in include/twq.h); ``twq`` is its thin
Python binding.
"""
from . import twq  # noqa: F401

__all__ = ["twq"]
