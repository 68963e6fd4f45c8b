"""Seeded synthetic workloads for windowed low-bit GDN / KDA decode.

This package is the only code that both the CUDA path and the CPU oracle see: it holds the
named workload shapes and the seeded input generators, and none of the method's arithmetic.
"""
from .configs import WORKLOADS, Workload, get  # noqa: F401
from .generate import (  # noqa: F401
    StepInputs,
    decode_inputs,
    outlier_scales,
    step_inputs,
    torch_dtype,
)
