"""B200-native W4A16 linear layer with a per-token-gated low-rank Error Compensator.

The compute lives in the CUDA shared library ``libspear.so`` (C ABI declared in
``include/spear.h``); ``w4_gemm_gated_b200.spear`` is its ctypes binding.
Importing this package does not load the library; importing the binding does,
and raises if the library is missing.
"""
__all__ = ["synth"]
