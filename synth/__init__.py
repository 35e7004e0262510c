"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This package holds input generation only: random draws, scaling of the draws
and rounding of fp32 draws to bf16 bit patterns.  It contains none of the
operator's arithmetic, so both the fp64 oracle and the CUDA library can be fed
from it without sharing any code with each other.
"""
from .inputs import (  # noqa: F401
    WORKLOAD_SHAPES,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    make_cmodal_inputs,
    make_fir_inputs,
    make_workload_inputs,
    make_modal_inputs,
)
