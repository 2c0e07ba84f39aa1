"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This package holds no arithmetic of the encoder itself: it only draws weights,
token ids and sequence lengths from seeded generators, and rounds parameters to
bf16-representable values when a workload asks for bf16 weights.
"""
from .albert_inputs import (  # noqa: F401
    ARCH,
    PARAM_ORDER,
    WORKLOADS,
    Workload,
    bf16_round,
    make_batch,
    make_weights,
    param_shapes,
)
