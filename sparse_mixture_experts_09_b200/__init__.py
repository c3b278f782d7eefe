"""B200-native Mixtral sparse-MoE feed-forward layer.

The layer runs in hand-written sm_100a CUDA kernels behind the C-ABI library
``libmoe.so`` (declared in ``include/moe.h``); ``moe`` is its ctypes binding,
``workloads`` and ``synth`` draw the seeded synthetic inputs.
"""
