"""B200-native (sm_100a) sparse MoE FFN layer forward behind a small C ABI.

The compute lives in the CUDA library libmoe_b200.so (built by
``python -m sparse_mixture_experts_21_b200.build``); ``_lib`` binds its entry
points, ``layer.MoELayer`` sequences them (bf16, fp32, fine-grained FP8 or MXFP8
experts; token- or expert-choice routing; CUDA-graph capture), ``ep.EPMoELayer``
shards the experts over ranks, ``replicas`` holds the data-parallel helpers and
``synth`` draws seeded inputs.
"""
from . import _lib, synth  # noqa: F401

__all__ = ["_lib", "synth"]
