"""GPU parity of the lightning indexer's KL-loss backward (sa_indexer_kl_grad) against
the float64 oracle (aclnnSparseLightningIndexerGradKLLoss, "Formula"), every element:
64 heads x 128 dims with 256 slots (BSND, two sequences) and 32 x 64 with 128 slots
(TND, three sequences).  dq / dk are bf16 (the bf16 rule of the parity harness), dw and
the loss fp32 (relative 2e-3 of the largest value)."""

import numpy as np
import pytest
import torch

from gen import make_indexer_inputs
from gen.torch_io import to_torch
from gpu_harness import bf16_bits, check_close, widen
from oracle.indexer_ref import IndexerProblem, indexer_kl_grad
from top_sparse_attention_attn_b200 import indexer_kl_grad as gpu_indexer_kl_grad

pytestmark = pytest.mark.gpu

CASES = {
    "h64_d128_bsnd": dict(seed=71, lens=(300, 300), H=64, d=128, topk=256, layout="BSND"),
    "h32_d64_tnd": dict(seed=72, lens=(200, 57, 130), H=32, d=64, topk=128, layout="TND"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_indexer_kl_grad_all_elements(name):
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for -m gpu tests")
    c = CASES[name]
    inp = make_indexer_inputs(**c)
    lens, H, d, topk = inp["lens"], c["H"], c["d"], c["topk"]
    pr = IndexerProblem(q=inp["q"], k=inp["k"], w=inp["w"], idx=inp["idx"], p=inp["p"], q_lens=lens,
                        kv_lens=lens, topk_len=inp["topk_len"])
    ref = indexer_kl_grad(pr)
    t = to_torch({k: v for k, v in inp.items() if isinstance(v, np.ndarray)}, "cuda")
    if c["layout"] == "BSND":
        B, S = len(lens), lens[0]
        loss, dq, dk, dw = gpu_indexer_kl_grad(t["q"].reshape(B, S, H, d), t["k"].reshape(B, S, d),
                                               t["w"].reshape(B, S, H), t["idx"].reshape(B, S, topk),
                                               t["p"].reshape(B, S, topk), topk_len=t["topk_len"].reshape(B, S))
    else:
        loss, dq, dk, dw = gpu_indexer_kl_grad(t["q"], t["k"], t["w"], t["idx"], t["p"], topk_len=t["topk_len"],
                                               cu_seqlens_q=t["cu_seqlens"], cu_seqlens_kv=t["cu_seqlens"])
    torch.cuda.synchronize()
    T = pr.T
    check_close(f"{name}:dq", widen(bf16_bits(dq)).reshape(T, -1), ref["dq"].reshape(T, -1))
    check_close(f"{name}:dk", widen(bf16_bits(dk)).reshape(-1), ref["dk"].reshape(-1))
    got_dw, got_loss = dw.cpu().numpy().reshape(T, H), loss.cpu().numpy().reshape(T)
    assert np.abs(got_dw - ref["dw"]).max() <= 2e-3 * np.abs(ref["dw"]).max(), name
    assert np.abs(got_loss - ref["loss"]).max() <= 2e-3 * np.abs(ref["loss"]).max() + 1e-6, name
