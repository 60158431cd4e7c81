"""B200-native forward pass of one token-choice Mixture-of-Experts FFN layer.

The compute runs in ``libmoe.so`` (hand-written sm_100a CUDA kernels behind a
C ABI, declared in ``include/moe.h``); ``mixture_experts_layer_51_b200.moe``
is the thin ctypes binding.  Importing the package loads nothing; the first
call into the binding loads the library and raises if it was not built.
"""
