"""B200-native (sm_100a) BCJR forward-backward sum-product over a bitshift trellis.

The compute lives in ``libbcjr.so`` (hand-written CUDA behind a C ABI declared in
``include/bcjr.h``); :mod:`bcjr_sum_product_b200.lib` is the thin ctypes binding.
Importing this package does not load the library; the first call does, and it
raises if the library has not been built.
"""
__all__ = ["lib", "inputs"]
