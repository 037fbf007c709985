"""The oracle reads fp16 inputs exactly (SparseFlashMlaGrad, "Parameter Description":
query, out, dOut and the KV inputs may be FLOAT16).

Every fp16 value is a float64 value, so a problem given as float16 arrays must give
bit-identical oracle results to the same values given as float64 arrays; the fp16
GPU parity test relies on it.
"""

import numpy as np

import oracle
from gen import make_inputs, scaled
from oracle.sparse_attn_ref import as_f64


def _f16(w, seed):
    inp = make_inputs(w)
    rng = np.random.default_rng(seed)
    for key in ("q", "k", "v", "kv", "cmp_kv", "do"):
        if key in inp:
            inp[key] = rng.standard_normal(inp[key].shape).astype(np.float16)
    return inp


def test_fp16_values_widen_exactly():
    x = np.array([np.float16(v) for v in (0.0, -0.0, 1.0, 6.1e-5, 5.96e-8, 65504.0, -3.14159, 0.1)])
    y = as_f64(x)
    assert y.dtype == np.float64
    np.testing.assert_array_equal(y.astype(np.float16), x)      # round trip
    np.testing.assert_array_equal(y, x.astype(np.float64))


def test_fp16_and_float64_inputs_give_identical_results():
    for w in (scaled("cfg1", "f16p", S=96, Hq=4, Hkv=2, block_size=16, topk=3, seed=71),
              scaled("cfg4", "f16p", seqlens=(40, 23), Hq=4, d_qk=64, d_v=64, cmp_topk=8, cmp_len_range=(4, 8),
                     win_left=9, seed=72)):
        a = _f16(w, seed=w.seed)
        b = {k: (v.astype(np.float64) if v.dtype == np.float16 else v) for k, v in a.items()}
        pa, pb = oracle.Problem.from_inputs(w, a), oracle.Problem.from_inputs(w, b)
        Oa, la = oracle.forward(pa, rounded=False)
        Ob, lb = oracle.forward(pb, rounded=False)
        np.testing.assert_array_equal(Oa, Ob)
        np.testing.assert_array_equal(la, lb)
        T = w.T
        ra = oracle.backward(pa, Oa, la, a["do"].reshape(T, w.Hq, w.d_v), rounded=False)
        rb = oracle.backward(pb, Ob, lb, b["do"].reshape(T, w.Hq, w.d_v), rounded=False)
        for key in ra:
            np.testing.assert_array_equal(ra[key], rb[key])
