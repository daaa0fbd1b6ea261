"""Seeded synthetic inputs shaped like the dynamic-sparse-attention workloads.

This package only draws random tensors and adds the planted structure that
makes attention sparse (a shared direction ``u`` on chosen key blocks, key
columns or diagonals).  It contains none of the method's arithmetic: no
pooling, scoring, selection or attention.  Both the CUDA library's tests and
the fp64 oracle consume the exact bf16 tensors produced here.
"""

from .workloads import (  # noqa: F401
    CONFIGS,
    Workload,
    DecodeWorkload,
    make_prefill,
    make_decode,
    planted_count,
    to_f64,
)
