"""Seeded synthetic inputs shared by the CUDA path, the oracle and the benchmark.

This package holds no attention arithmetic. It only turns (seed, shape) into
bf16 tensors, so that the CUDA library and the CPU oracle can be fed the same
bytes without either one depending on the other.
"""
from .gen import (  # noqa: F401
    GAMMA,
    splitmix64,
    normal_bf16,
    uniform_f32,
    peaky_positions,
    workload,
    WORKLOADS,
)
