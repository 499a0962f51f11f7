"""Seeded synthetic inputs for the BitLinear forward.

This package only draws random numbers and rounds them to the storage type
the workload asks for.  It holds none of the method's arithmetic (no
quantisation, no packing, no contraction), so both the CPU oracle and the
CUDA path may take their inputs from it.
"""

from .gen import (  # noqa: F401
    CONFIGS,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    rng_for,
    latent_weights,
    acts_normal,
    acts_normal_outliers,
    acts_student_t,
    config_inputs,
    layer_weights,
    PROJECTIONS,
)
