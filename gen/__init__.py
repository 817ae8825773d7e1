"""Seeded synthetic inputs for HSTU jagged attention and the HSTU layer.

This package only draws random numbers and lays them out. It holds none of
the method's arithmetic (no scores, no SiLU, no bucketing, no normalisation),
so both the fp64 oracle and the CUDA path can consume its output without
sharing any computation.
"""

from .hstu_inputs import (  # noqa: F401
    CONFIGS,
    AttnInputs,
    LayerInputs,
    make_attn_inputs,
    make_layer_inputs,
    make_inputs,
    round_to_bf16,
    custom_attn_inputs,
    take_sequences,
)
