"""Seeded synthetic inputs for the attention forward, shared by the tests and the bench.

This module holds no attention arithmetic: it only draws random tensors, builds
integer length tables and boolean structure (a causal mask tensor), and lists
the workload shapes.  Both the float64 oracle and the CUDA path consume what it
returns; neither is imported here.
"""
from .gen import (  # noqa: F401
    normal,
    varlen_lengths,
    cumulative,
    causal_mask_u8,
    alibi_slopes,
    TORCH_DTYPES,
)
from .configs import CONFIGS, Workload, build  # noqa: F401
