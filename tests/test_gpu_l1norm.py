"""GPU parity of the SoftmaxL1Norm outputs (sa_softmax_l1norm) against the oracle.

SparseFlashMlaGrad, "Parameter Description" (oriSoftmaxL1NormOptional /
cmpSoftmaxL1NormOptional) with the target distribution of
aclnnSparseLightningIndexerGradKLLoss, "Formula".  Both sides take the same lse
(the oracle's forward, rounded to fp32, or the GPU forward's at full size), so
the comparison isolates this output.  Tolerance: the GPU sums fp32 exponentials of
fp32-accumulated bf16 scores; relative 2e-3 with an absolute floor of 1e-5 on
values that are probabilities (each row sums to 1).
"""

import numpy as np
import pytest
import torch

import oracle
from gen import get_workload, make_inputs, scaled
from gpu_harness import device_problem

pytestmark = pytest.mark.gpu

CASES = {
    "cfg1_full": (get_workload("cfg1"), {}),                                     # blocks of 64
    "cfg2_future_len": (scaled("cfg2", "future", S=448, Hq=16, Hkv=1, seed=22),
                        dict(allow_future=True, ori_len_range=(0, 16))),
    "cfg5_empty_rows": (scaled("cfg5", "empty", S=512, Hq=8, Hkv=2, p_drop=0.6, seed=27), {}),
    "block_bs16_d64": (scaled("cfg1", "bs16", S=300, Hq=8, Hkv=2, block_size=16, topk=6, seed=29), {}),
    "block_bs128_d64": (scaled("cfg1", "bs128", S=600, Hq=4, Hkv=1, block_size=128, topk=3, seed=30), {}),
    "block_tnd": (scaled("cfg1", "tnd", layout="TND", seqlens=(200, 64, 333), Hq=8, Hkv=1, seed=31), {}),
    "cfg3_small": (scaled("cfg3", S=700, Hq=32, topk=256, seed=23), {}),
    "token_h64_topk": (scaled("cfg3", "h64", S=400, Hq=64, topk=256, seed=35), {}),
    "cfg4_small": (scaled("cfg4", seqlens=(100, 300, 37), Hq=16, cmp_topk=64, cmp_len_range=(16, 64),
                          seed=24), {}),
}


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for -m gpu tests")


def _compare(name, got, ref):
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), name
    np.testing.assert_allclose(got, ref, rtol=2e-3, atol=1e-5, err_msg=name)
    sums = got.sum(axis=-1)
    assert np.all((np.abs(sums - 1) < 1e-4) | (np.abs(sums) < 1e-6)), name


@pytest.mark.parametrize("name", list(CASES))
def test_softmax_l1norm_all_elements(name):
    _need_gpu()
    w, kw = CASES[name]
    inputs = make_inputs(w, **kw)
    p = oracle.Problem.from_inputs(w, inputs)
    _, lse_ref = oracle.forward(p)                       # fp32
    ref_ori, ref_cmp = oracle.softmax_l1norm(p, lse_ref)
    sa, _ = device_problem(w, inputs)
    lse = torch.from_numpy(np.ascontiguousarray(lse_ref.reshape(sa._lead() + (w.Hq,)))).cuda()
    ori, cmp = sa.softmax_l1norm(lse)
    torch.cuda.synchronize()
    assert (ori is None) == (ref_ori is None) and (cmp is None) == (ref_cmp is None), name
    if ori is not None:
        _compare(f"{name}:ori", ori.cpu().numpy().reshape(ref_ori.shape), ref_ori)
    if cmp is not None:
        _compare(f"{name}:cmp", cmp.cpu().numpy().reshape(ref_cmp.shape), ref_cmp)


def test_softmax_l1norm_full_size_sampled():
    """cfg2 at full size in one call; the oracle checks 24 sampled units on the GPU lse."""
    _need_gpu()
    w = get_workload("cfg2")
    inputs = make_inputs(w)
    p = oracle.Problem.from_inputs(w, inputs)
    sa, _ = device_problem(w, inputs)
    _, lse = sa.forward()
    ori, _ = sa.softmax_l1norm(lse)
    torch.cuda.synchronize()
    got = ori.cpu().numpy().reshape(w.T, w.Hkv, -1)
    lse_h = lse.cpu().numpy().reshape(w.T, w.Hq)
    rng = np.random.default_rng(5)
    units = [(int(t), int(g)) for t, g in zip(rng.integers(0, w.T, 24), rng.integers(0, w.Hkv, 24))]
    ref, _ = oracle.softmax_l1norm(p, lse_h, units=units)
    for tq, g in units:
        _compare(f"cfg2:{tq},{g}", got[tq, g], ref[tq, g])
