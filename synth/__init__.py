"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This package holds no arithmetic of the encoder itself: it only draws weights,
token ids, sequence lengths, duration logits and token features from seeded
generators, and rounds values to bf16-representable ones where a workload asks.
"""
from .albert_inputs import (  # noqa: F401
    ARCH,
    DURATION_CHANNELS,
    LAYER_PARAMS,
    PARAM_ORDER,
    WORKLOADS,
    Workload,
    bf16_round,
    make_batch,
    make_duration_logits,
    make_features,
    make_weights,
    param_shapes,
)
