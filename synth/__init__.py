"""Seeded synthetic inputs shared by the oracle and the CUDA path.

This package holds shapes, seeded random weights and prompts, and nothing of
the looped model's arithmetic. Both the oracle (``oracle/``) and the CUDA
binding read their inputs from here; neither imports the other.
"""
from .inputs import (  # noqa: F401
    Shape,
    TINY,
    TINY_BF16,
    DORY_4B,
    SMALL128,
    SHAPES,
    layer_kinds,
    weight_specs,
    make_weights,
    make_prompt,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
)
