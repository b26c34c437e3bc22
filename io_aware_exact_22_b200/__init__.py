"""Exact fused attention (FlashAttention forward and backward) for NVIDIA B200, sm_100a.

The compute path lives in ``libfa.so`` (hand-written CUDA kernels behind a C ABI, see
``include/fa.h``).  ``io_aware_exact_22_b200.fa`` is the thin ctypes binding over that ABI.
Importing this package does not load the library; the first call through ``fa`` does, and
fails loudly when the library is missing.
"""
