"""Seeded synthetic inputs for the full-vocabulary distillation loss.

This package only draws random numbers and shapes them into hidden states,
unembedding matrices and labels. It holds none of the loss arithmetic, so both
the CPU oracle and the CUDA library can be fed from it without sharing code.
"""

from .workloads import (  # noqa: F401
    IGNORE_INDEX,
    WORKLOADS,
    Inputs,
    PROFILE_WORKLOADS,
    Workload,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    gaussian_bf16,
    matrix_with_spectrum,
    make_inputs,
    make_custom,
)
