"""B200-native (sm_100a) forward pass of a token-choice top-k Mixture-of-Experts layer.

The compute lives in libmoe_b200.so (C ABI, include/moe.h); `moe` is its Python
binding and `layer.MoELayer` sequences the calls.  `inputs` generates seeded
synthetic workloads.
"""
from . import inputs  # noqa: F401

__all__ = ["inputs", "moe", "layer"]


def __getattr__(name):
    # the binding and layer import torch and load the CUDA library lazily
    if name in ("moe", "layer"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
