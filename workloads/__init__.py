"""Seeded synthetic inputs and workload shapes for the FP8 W8A8 linear path.

This package is the one thing the CUDA path and the CPU oracle share. It holds
random-number generation, bit packing of the input formats and the workload
shapes, and none of the method's arithmetic: no scale rule, no FP8 encoding,
no GEMM.
"""

from .generators import (
    activations_bf16,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    moe_routing,
    q4_weights,
)
from .configs import CONFIGS, DecodeShapes, workload

__all__ = [
    "activations_bf16",
    "bf16_bits_to_f32",
    "f32_to_bf16_bits",
    "moe_routing",
    "q4_weights",
    "CONFIGS",
    "DecodeShapes",
    "workload",
]
