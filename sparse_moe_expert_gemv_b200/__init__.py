"""B200-native (sm_100a) sparse MoE expert layer.

The compute lives in ``libmoe.so`` (CUDA kernels behind the C ABI of
``include/moe.h``); ``binding`` is its ctypes binding.  ``inputs`` draws the
seeded synthetic workloads.  Importing ``binding`` fails loudly when the
library has not been built.
"""
