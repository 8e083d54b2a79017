"""Seeded synthetic inputs for the token-sparse decode step.

This package is shared by the CUDA path's tests and benchmark and by the
oracle's tests.  It draws random numbers, rotates keys and queries into their
post-RoPE form (that is how a model writes its cache, before any decode step
runs) and rounds them to bf16.  It holds none of the decode step's own
arithmetic: no importance score, no selection, no attention.
"""

from .synth import (  # noqa: F401
    ROLE_SPARSE,
    ROLE_DENSE,
    ROLE_STREAM,
    WorkloadSpec,
    Workload,
    PRESETS,
    preset,
    make_workload,
    rope_rotate_f32,
    token_draws,
    HeadWeightSpec,
    HEAD_WEIGHT_PRESETS,
    head_weights,
)
