"""Seeded synthetic inputs for the Prox sparse SwiGLU FFN decode step.

This module only draws random numbers and rounds them to bf16 storage; it holds
none of the method's arithmetic.  Both the fp64 oracle tests and the CUDA path
take their inputs from here, so the two sides always see the same values.
"""

from .configs import CONFIGS, WorkloadConfig, ffn_k, get_config
from .layers import (
    SyntheticLayer,
    bf16_round,
    bf16_bits_to_f32,
    make_layer,
    make_stack_layer,
    outlier_channels,
)

__all__ = [
    "CONFIGS",
    "WorkloadConfig",
    "ffn_k",
    "get_config",
    "SyntheticLayer",
    "bf16_round",
    "bf16_bits_to_f32",
    "make_layer",
    "make_stack_layer",
    "outlier_channels",
]
