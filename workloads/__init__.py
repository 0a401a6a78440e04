"""Seeded synthetic inputs shared by the tests of both the CUDA path and the oracle."""
from .synth import (AWQ_GRID, C1, C2, C3, C4, C5, CONFIGS, LayerSpec, bf16_bits_from_f32,
                    bf16_bits_to_f32, bf16_bits_to_f64, channel_gains, make_channel_scales,
                    make_weight, make_x_bits, small_spec)

__all__ = ["AWQ_GRID", "C1", "C2", "C3", "C4", "C5", "CONFIGS", "LayerSpec",
           "bf16_bits_from_f32", "bf16_bits_to_f32", "bf16_bits_to_f64", "channel_gains",
           "make_channel_scales", "make_weight", "make_x_bits", "small_spec"]
