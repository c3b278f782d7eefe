"""B200-native Mixtral sparse-MoE feed-forward layer.

The layer runs in hand-written sm_100a CUDA kernels behind the C-ABI library
``libmoe.so`` (declared in ``include/moe.h``); ``moe`` is its ctypes binding,
``workloads`` and ``synth`` draw the seeded synthetic inputs.
"""
__all__ = ["moe", "synth", "workloads"]


def __getattr__(name):
    if name == "moe":
        from . import moe
        return moe
    raise AttributeError(name)
