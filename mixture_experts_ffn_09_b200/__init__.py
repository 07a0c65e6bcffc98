"""libmoe: a B200-native top-k mixture-of-experts FFN forward.

The compute lives in ``libmoe.so`` (CUDA C++ for sm_100a behind a C ABI,
declared in ``include/moe.h``); ``mixture_experts_ffn_09_b200.moe`` is the
thin ctypes binding.  Importing the package does not load the library;
calling into the binding does, and fails loudly when it is missing.
"""
__all__ = ["synth"]
