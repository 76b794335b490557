"""Seeded synthetic inputs shared by the CPU oracle, the GPU tests and the bench.

This package draws random numbers and lays out arrays; it holds none of the
SVDQuant arithmetic (no smoothing, factorisation or quantisation), so that the
oracle and the CUDA path can both consume it without sharing method code.
"""

from .workloads import (  # noqa: F401
    Workload,
    WORKLOADS,
    make_workload,
    make_case,
    generate,
    to_bf16,
    bf16_bits_to_f32,
)
