"""Packed 1-bit / balanced-ternary matmul for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libbnn.so`` (hand-written CUDA) and
its thin binding ``ternary_neural_net_b200.bnn``.  Importing this package does
not load the library; ``from ternary_neural_net_b200 import bnn`` does, and
fails loudly when it is missing.
"""
import importlib

__all__ = ["bnn", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
