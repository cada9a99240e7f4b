"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and bench.py.

This module holds no step of the attention method: it only draws numbers.
"""
from .fourier_field import (  # noqa: F401
    WORKLOADS,
    Workload,
    make_inputs,
    to_bf16_tensor,
)
