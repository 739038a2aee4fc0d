"""Seeded synthetic inputs shared by the CUDA path's tests, the oracle's tests and bench.py.

This package draws random numbers and lays them out; it holds none of the
method's arithmetic (no counting, no placement, no planning, no combine).
Both sides of every parity test receive the same arrays from here.
"""
from .workloads import (  # noqa: F401
    Workload,
    WORKLOADS,
    make_routing,
    make_gates,
    make_hidden,
    make_expert_scales,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
)
