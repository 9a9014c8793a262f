"""Seeded synthetic inputs shared by the GPU path's tests/bench and by the oracle.

This module only draws numbers: it holds none of the GEMM's arithmetic.
"""
from .gen import (  # noqa: F401
    BASE_SEED,
    bf16_bits_to_f64,
    f16_bits_to_f64,
    f64_to_bf16_bits,
    f64_to_f16_bits,
    matrix_bf16,
    matrix_f16,
    normal_f64,
    seed_for,
    splitmix64,
    uniform01_f64,
)
