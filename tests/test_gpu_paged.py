"""GPU parity of the forward over a paged KV cache (aclnnNsaSelectedAttentionInfer:
"paged attention obtains the kvCache", a few query tokens per sequence) against the
oracle, element by element: NSA block selection (192 / 128, generic kernels),
token-level selection over a shared 576 / 512 row with 64 heads (the tcgen05 token
forward, its TMA row gathers following the block table) and 16-row blocks."""

import numpy as np
import pytest
import torch

import oracle
from gen import make_paged_inputs
from gen.torch_io import to_torch
from gpu_harness import bf16_bits, check_close, check_lse, widen
from top_sparse_attention_attn_b200 import SparseAttention
from top_sparse_attention_attn_b200 import _lib as L

pytestmark = pytest.mark.gpu

CASES = {
    "nsa_block_192": dict(seed=61, B=8, s_q=2, kv_lens=(300, 1111, 64, 2999, 777, 130, 1600, 2048), page=64,
                          Hq=16, Hkv=1, d_qk=192, d_v=128, kv_shared=False, block_size=64, topk=16),
    "token_576_h64": dict(seed=62, B=4, s_q=4, kv_lens=(300, 1500, 97, 2048), page=128, Hq=64, Hkv=1,
                          d_qk=576, d_v=512, kv_shared=True, block_size=1, topk=256),
    "block16_d64": dict(seed=63, B=5, s_q=3, kv_lens=(50, 400, 1000, 17, 256), page=32, Hq=8, Hkv=2,
                        d_qk=64, d_v=64, kv_shared=False, block_size=16, topk=8),
}


def _problem(inp):
    m = inp["_meta"]
    B, s_q = m["B"], m["s_q"]
    if m["kv_shared"]:
        k = inp["kv"]
        v = inp["kv"][..., :m["d_v"]]
    else:
        k, v = inp["k"], inp["v"]
    return oracle.Problem(q=inp["q"], k_ori=k, v_ori=v, kv_shared=m["kv_shared"], q_lens=[s_q] * B,
                          kv_lens=[m["s_kv"]] * B, Hq=m["Hq"], Hkv=m["Hkv"], d_qk=m["d_qk"], d_v=m["d_v"],
                          scale=m["d_qk"] ** -0.5, block_size=m["block_size"],
                          ori_idx=inp["ori_idx"].astype(np.int64), sinks=inp.get("sinks"),
                          kv_used=inp["seqused_kv"], block_table=inp["block_table"], page_size=m["page"])


def _device(inp):
    m = inp["_meta"]
    t = to_torch({k: v for k, v in inp.items() if k != "_meta"}, "cuda")
    B, s_q = m["B"], m["s_q"]
    kw = dict(layout="BSND", Hq=m["Hq"], Hkv=m["Hkv"], d_qk=m["d_qk"], d_v=m["d_v"], scale=m["d_qk"] ** -0.5,
              q=t["q"].reshape(B, s_q, m["Hq"], m["d_qk"]), kv_shared=m["kv_shared"], block_size=m["block_size"],
              batch=B, s_q=s_q, s_kv=m["s_kv"], t_kv=m["t_kv"],
              ori_idx=t["ori_idx"].reshape(B, s_q, m["Hkv"], m["topk"]), seqused_kv=t["seqused_kv"],
              block_table=t["block_table"], page_size=m["page"], sinks=t.get("sinks"))
    if m["kv_shared"]:
        kw["kv"] = t["kv"]
    else:
        kw["k"], kw["v"] = t["k"], t["v"]
    return SparseAttention(**kw)


@pytest.mark.parametrize("name", list(CASES))
def test_paged_forward_all_elements(name):
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for -m gpu tests")
    inp = make_paged_inputs(**CASES[name])
    p = _problem(inp)
    O_ref, lse_ref = oracle.forward(p)
    sa = _device(inp)
    o, lse = sa.forward()
    torch.cuda.synchronize()
    T = p.T
    check_close(f"{name}:O", widen(bf16_bits(o)).reshape(T, -1), widen(O_ref).reshape(T, -1))
    check_lse(f"{name}:lse", lse.cpu().numpy().reshape(T, -1), lse_ref)
    # the backward is not defined over a paged cache
    import ctypes
    n = ctypes.c_size_t(0)
    assert L.lib().sa_bwd_get_workspace_size(ctypes.byref(sa.args()), ctypes.byref(n)) == L.SA_ERR_UNSUPPORTED
