"""Seeded synthetic inputs for the W4 + gated error-compensator linear layer.

This package only draws random numbers and rounds them to the storage types the
layer takes (bf16 activations and EC factors, fp32 master weights).  It holds
none of the layer's arithmetic, so the CPU oracle and the CUDA path can both be
fed from it without sharing any code of the method.
"""
from .workloads import (  # noqa: F401
    Layer,
    bf16_bits_from_f32,
    f32_from_bf16_bits,
    make_layer,
    config_layers,
    CONFIG_NAMES,
    CONFIG_M,
)
