"""The torch binding's host-side checks (no GPU): the element type it passes through
the C ABI, which cannot see tensor types behind its raw pointers."""

import pytest
import torch

from top_sparse_attention_attn_b200 import SparseAttention
from top_sparse_attention_attn_b200 import _lib as L


def _problem(dtype_q, dtype_kv):
    T, Hq, Hkv, d = 8, 4, 2, 64
    return SparseAttention(layout="TND", Hq=Hq, Hkv=Hkv, d_qk=d, d_v=d, scale=0.125,
                           q=torch.zeros(T, Hq, d, dtype=dtype_q),
                           k=torch.zeros(T, Hkv, d, dtype=dtype_kv), v=torch.zeros(T, Hkv, d, dtype=dtype_kv),
                           t_q=T, t_kv=T, block_size=1,
                           ori_idx=torch.zeros(T, Hkv, 2, dtype=torch.int32),
                           cu_seqlens_q=torch.tensor([0, T], dtype=torch.int32),
                           cu_seqlens_kv=torch.tensor([0, T], dtype=torch.int32))


@pytest.mark.parametrize("dtype,code", [(torch.bfloat16, L.SA_DTYPE_BF16), (torch.float16, L.SA_DTYPE_FP16)])
def test_element_type_follows_the_tensors(dtype, code):
    assert _problem(dtype, dtype).args().dtype == code


def test_mixed_or_unsupported_element_types_are_rejected():
    with pytest.raises(TypeError):
        _problem(torch.float16, torch.bfloat16).args()
    with pytest.raises(TypeError):
        _problem(torch.float32, torch.float32).args()
