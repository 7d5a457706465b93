"""B200-native (sm_100a) sparse MoE FFN layer forward behind a small C ABI.

The compute lives in the CUDA library libmoe_b200.so (built by
``python -m sparse_mixture_experts_21_b200.build``); ``_lib`` binds its entry
points, ``layer.MoELayer`` sequences them, ``synth`` draws seeded inputs.
"""
from . import _lib, synth  # noqa: F401

__all__ = ["_lib", "synth"]
