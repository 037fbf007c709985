"""GPU parity for fp16 inputs (SparseFlashMlaGrad, "Parameter Description": q, k, v,
dO and the gradients are BFLOAT16 or FLOAT16, the outputs of the inputs' type).

fp16 problems run on the generic query-stationary kernels with fp16 MMA operands
and fp32 accumulation.  The inputs are drawn at full fp16 precision (most values
are not bf16-representable), and the float64 oracle reads exactly those values.

Tolerances, from fp16's unit roundoff u = 2^-11: O within 5u of max|O| (P and O
are each rounded to fp16 once, everything else accumulates in fp32); dQ / dK /
dV / dCmpKv within 10u of their max|ref| (dS and P rounded to fp16, then fp32
sums over the selected rows); lse within 1e-4 absolute; the cosine to the
reference >= 1 - 1e-5.  A path that rounded the fp16 operands to bf16 (u = 2^-8)
would miss these bounds.
"""

import numpy as np
import pytest
import torch

import oracle
from gen import make_inputs, scaled
from gen.torch_io import to_torch
from top_sparse_attention_attn_b200 import SparseAttention
from top_sparse_attention_attn_b200 import _lib as L

pytestmark = pytest.mark.gpu

U = 2.0 ** -11

CASES = {
    # block-level, 64-row blocks at d 192/128 (the bf16 fast paths' shape) and 16-row blocks at d 64
    "block_192_128": (scaled("cfg2", "f16", S=320, Hq=16, Hkv=2, topk=4, seed=61), {}),
    "block_bs16_d64": (scaled("cfg1", "f16", S=300, Hq=8, Hkv=2, block_size=16, topk=6, seed=62), {}),
    # token-level over one shared 576/512 KV head, 64 heads per kv-head
    "token_576_h64": (scaled("cfg3", "f16", S=200, Hq=64, topk=64, seed=63), {}),
    # window over the original KV + top-k compressed rows + sinks, TND
    "swa_cmp_sinks": (scaled("cfg4", "f16", seqlens=(100, 37), Hq=16, cmp_topk=32, cmp_len_range=(8, 32),
                             seed=64), {}),
}

_FLOAT_KEYS = ("q", "k", "v", "kv", "cmp_kv", "do")


def _fp16_inputs(w, kw, seed):
    """The workload's indices, lengths and sinks, with fresh fp16 float tensors."""
    inp = make_inputs(w, **kw)
    rng = np.random.default_rng(seed)
    for key in _FLOAT_KEYS:
        if key in inp:
            scale = w.do_scale if key == "do" else 1.0
            inp[key] = (rng.standard_normal(inp[key].shape) * scale).astype(np.float16)
    return inp


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def _close(name, got, ref, rel):
    got, ref = np.asarray(got, np.float64).ravel(), np.asarray(ref, np.float64).ravel()
    assert got.shape == ref.shape, name
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    mref = np.abs(ref).max()
    err = np.abs(got - ref).max()
    assert err <= rel * mref + 1e-30, f"{name}: max|err| {err:.4g} > {rel:.3g} * max|ref| {mref:.4g}"
    nr, ng = np.linalg.norm(ref), np.linalg.norm(got)
    if nr > 0:
        assert got @ ref / (nr * ng) >= 1 - 1e-5, f"{name}: cosine"


@pytest.mark.parametrize("name", list(CASES))
def test_fp16_forward_backward_against_the_oracle(name):
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for -m gpu tests")
    w, kw = CASES[name]
    inp = _fp16_inputs(w, kw, seed=w.seed + 1000)
    p = oracle.Problem.from_inputs(w, inp)
    T = w.T
    t = to_torch(inp, "cuda")
    assert t["q"].dtype == torch.float16
    sa = SparseAttention.from_workload(w, t)
    assert sa.plan() == (L.SA_KERNEL_FWD_GENERIC, L.SA_KERNEL_BWD_GENERIC)

    O_ref, lse_ref = oracle.forward(p, rounded=False)
    ws = sa.fwd_workspace()
    o, lse = sa.forward(ws=ws)
    torch.cuda.synchronize()
    assert o.dtype == torch.float16
    assert sa.read_status(ws) == 0
    _close(f"{name}:O", _f64(o).reshape(T, -1), O_ref.reshape(T, -1), 5 * U)
    l_ref = lse_ref.reshape(T, -1)
    fin = np.isfinite(l_ref)
    assert np.array_equal(fin, np.isfinite(lse.cpu().numpy().reshape(T, -1)))
    assert np.abs(lse.cpu().numpy().reshape(T, -1)[fin] - l_ref[fin]).max() <= 1e-4

    # the backward on the GPU's own O and lse (fp16 O, as a caller would pass it)
    do = inp["do"].reshape(T, w.Hq, w.d_v)
    O16 = _f64(o).reshape(T, w.Hq, w.d_v)
    ref = oracle.backward(p, O16, lse.cpu().numpy().astype(np.float64).reshape(T, w.Hq), do, rounded=False)
    wsb = sa.bwd_workspace()
    grads = sa.backward(o, lse, t["do"], ws=wsb)
    torch.cuda.synchronize()
    assert sa.read_status(wsb) == 0
    for key, r in ref.items():
        if key == "dsinks":
            _close(f"{name}:dsinks", grads["dsinks"].cpu().numpy(), r, 10 * U)
            continue
        g = grads[key]
        assert g.dtype == torch.float16, key
        _close(f"{name}:{key}", _f64(g).reshape(r.shape[0], -1), r.reshape(r.shape[0], -1), 10 * U)


def test_fp16_softmax_l1norm_against_the_oracle():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for -m gpu tests")
    w, kw = CASES["swa_cmp_sinks"]
    inp = _fp16_inputs(w, kw, seed=77)
    p = oracle.Problem.from_inputs(w, inp)
    t = to_torch(inp, "cuda")
    sa = SparseAttention.from_workload(w, t)
    _, lse = sa.forward()
    _, cmp = sa.softmax_l1norm(lse)
    torch.cuda.synchronize()
    _, cmp_ref = oracle.softmax_l1norm(p, lse.cpu().numpy().astype(np.float64).reshape(w.T, w.Hq))
    _close("l1norm:cmp", cmp.cpu().numpy(), cmp_ref, 10 * U)
