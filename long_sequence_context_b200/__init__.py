"""long_sequence_context_b200: causal ring attention (context parallel,
zigzag 2N split, log-sum-exp merge, recompute backward) on one B200.

The computation lives in libcpattn.so (CUDA for sm_100a, C ABI in
include/cpattn.h); ``cpattn`` is its Python binding.
"""
__all__ = ["cpattn", "inputs"]
