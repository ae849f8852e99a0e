"""Exact IO-aware (FlashAttention-style) attention for one NVIDIA B200 (sm_100a).

The compute lives in the CUDA library built from ``csrc/`` (C ABI in
``include/fa.h``); ``fa`` is its Python binding, ``workloads`` the seeded
synthetic inputs.
"""
