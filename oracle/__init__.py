"""Float64 CPU oracle for top-k index-selected sparse attention.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
CPU-baseline leg of the benchmark; never by the CUDA product path.
"""

from .indexer_ref import IndexerProblem, indexer_kl_grad, indexer_slots, unit_indexer_kl
from .sparse_attn_ref import (Problem, backward, forward, round_to_bf16_bits, softmax_l1norm,
                              unit_backward, unit_flops, unit_forward, unit_softmax_l1norm,
                              visible_rows, widen_bf16)

__all__ = ["IndexerProblem", "indexer_kl_grad", "indexer_slots", "unit_indexer_kl", "Problem", "backward", "forward", "round_to_bf16_bits", "softmax_l1norm", "unit_backward",
           "unit_flops", "unit_forward", "unit_softmax_l1norm", "visible_rows", "widen_bf16"]
