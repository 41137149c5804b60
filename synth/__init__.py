"""Seeded synthetic inputs shared by the CUDA path's tests, the CPU oracle's tests and bench.py.

This package draws random numbers and rounds them to BF16.  It holds none of the
quantization or GEMM arithmetic: it produces bit patterns that both sides consume.

Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
as 1, 2, 3", SC 2011), keyed by (seed, stream) and addressed by a 64-bit counter, so that
any element of any tensor can be regenerated on its own (a row slice of a large matrix
equals the same rows of the full matrix).
"""
from .philox import philox4x32_10, uniform_open01, normal_pairs
from .workloads import (
    f64_to_bf16_bits, bf16_bits_to_f32, normal_bf16, uniform_bf16, student_t3_bf16,
    outlier_channels, WORKLOADS, workload,
)

__all__ = [
    "philox4x32_10", "uniform_open01", "normal_pairs",
    "f64_to_bf16_bits", "bf16_bits_to_f32", "normal_bf16", "uniform_bf16",
    "student_t3_bf16", "outlier_channels", "WORKLOADS", "workload",
]
