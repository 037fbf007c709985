"""Top-k index-selected sparse attention (forward + backward) for one NVIDIA B200.

The compute lives in libsparse_attn.so (CUDA, sm_100a) behind the C ABI of
include/sparse_attn.h; `_lib` is its ctypes binding and `api.SparseAttention`
a thin wrapper that marshals torch tensors into it.
"""

from . import _lib
from ._lib import SaError
from .api import SparseAttention, indexer_kl_grad

__all__ = ["SparseAttention", "SaError", "_lib", "indexer_kl_grad"]
