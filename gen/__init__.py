"""Seeded synthetic input generators shared by the oracle tests, the GPU tests and bench.py.

This package draws numbers only; it holds none of the fast-weight method's arithmetic.
"""

from . import rng, workloads  # noqa: F401
from .workloads import (  # noqa: F401
    INPLACE_128K_TARGET,
    INPLACE_4B,
    INPLACE_FP32,
    LINEAR_GD,
    SR_TTT_GATE,
    WORKLOADS,
    InplaceSpec,
    LinearSpec,
    inplace_inputs,
    linear_inputs,
    needle_positions,
    scaled,
)
