"""Seeded synthetic inputs for top-k index-selected sparse attention.

This package is shared by the float64 oracle tests, the GPU parity tests and the
benchmark.  It draws random tensors and index sets only; it contains none of the
attention arithmetic.
"""

from .configs import WORKLOADS, Workload, get_workload, scaled
from .synth import make_indexer_inputs, make_inputs, make_paged_inputs, bf16_bits_from_f32, f32_from_bf16_bits

__all__ = [
    "WORKLOADS",
    "Workload",
    "get_workload",
    "scaled",
    "make_inputs",
    "make_paged_inputs",
    "make_indexer_inputs",
    "bf16_bits_from_f32",
    "f32_from_bf16_bits",
]
