"""KDA (Kimi Delta Attention) forward for NVIDIA B200 (sm_100a).

The compute lives in a C-ABI CUDA library (``libkda_b200.so``, declared in
``include/kda.h``); ``kda_linear_attention_fwd_b200.kda`` is its thin ctypes
binding.  Importing this package does not load the library; the binding
loads it on first use and raises if it is missing.
"""
__all__ = ["kda", "workloads"]
