"""Pins for sequsedQ / sequsedOriKv / sequsedCmpKv in the oracle.

SparseFlashMlaGrad, "Parameter Description": the number of query, original-KV and
compressed-KV tokens of each batch that actually take part in the computation.
A padded problem with used lengths must give what the same problem gives with
each sequence cut to its used tokens (every index lies inside the used part), and
the rows past the used lengths must behave as rows that select nothing: O = 0,
lse from the sink alone (+inf without one), and zero gradients.
"""

import numpy as np
import pytest

import oracle
from oracle import Problem

LENS, USED = (13, 9), (9, 6)


def _spec(kind, seed):
    rng = np.random.default_rng(seed)
    T = sum(LENS)
    Hq, Hkv, d = 4, 2, 6
    spec = dict(kind=kind, Hq=Hq, Hkv=Hkv, d=d, q=rng.standard_normal((T, Hq, d)),
                kv=rng.standard_normal((T, Hkv, d)), v=rng.standard_normal((T, Hkv, d)),
                do=rng.standard_normal((T, Hq, d)), sinks=rng.standard_normal(Hq))
    if kind == "token":
        topk = 4
        idx = np.full((T, Hkv, topk), -1, dtype=np.int64)
        off = 0
        for L, U in zip(LENS, USED):
            for t in range(L):
                for g in range(Hkv):
                    hi = U if t < U else L                      # rows past sequsedQ may point anywhere
                    sel = rng.permutation(hi)[:rng.integers(0, topk + 1)]
                    idx[off + t, g, :len(sel)] = sel
            off += L
        spec["idx"] = idx
    elif kind == "block":
        bs, topk = 2, 3
        idx = np.full((T, Hkv, topk), -1, dtype=np.int64)
        off = 0
        for L, U in zip(LENS, USED):
            for t in range(L):
                for g in range(Hkv):
                    nb = (U if t < U else L) // bs
                    sel = rng.permutation(nb)[:rng.integers(1, topk + 1)]
                    idx[off + t, g, :len(sel)] = sel
            off += L
        spec["idx"], spec["bs"] = idx, bs
    elif kind == "swa_cmp":
        ratio, ctopk = 2, 3
        clens = tuple(L // ratio for L in LENS)
        cused = tuple(U // ratio for U in USED)
        cidx = np.full((T, Hkv, ctopk), -1, dtype=np.int64)
        off = 0
        for L, U, C, CU in zip(LENS, USED, clens, cused):
            for t in range(L):
                for g in range(Hkv):
                    hi = CU if t < U else C
                    sel = rng.permutation(hi)[:rng.integers(0, ctopk + 1)]
                    cidx[off + t, g, :len(sel)] = sel
            off += L
        spec.update(cidx=cidx, ratio=ratio, clens=clens, cused=cused,
                    ckv=rng.standard_normal((sum(clens), Hkv, d)))
    return spec


def _problem(spec, lens, cut):
    """The problem over `lens` (the padded lengths with used lengths, or the cut ones)."""
    kind, Hq, Hkv, d = spec["kind"], spec["Hq"], spec["Hkv"], spec["d"]
    rows = np.concatenate([np.arange(o, o + n) for o, n in zip(np.cumsum((0,) + LENS[:-1]), lens)])
    kw = dict(q_lens=lens, kv_lens=lens, Hq=Hq, Hkv=Hkv, d_qk=d, d_v=d, scale=0.6, sinks=spec["sinks"])
    if not cut:
        kw.update(q_used=USED, kv_used=USED)
    q = spec["q"][rows]
    if kind == "block":
        kw.update(k_ori=spec["kv"][rows], v_ori=spec["v"][rows], kv_shared=False, block_size=spec["bs"],
                  ori_idx=spec["idx"][rows])
    else:
        kv = spec["kv"][rows]
        kw.update(k_ori=kv, v_ori=kv, kv_shared=True)
        if kind == "token":
            kw["ori_idx"] = spec["idx"][rows]
        else:
            coffs = np.cumsum((0,) + spec["clens"][:-1])
            crows = np.concatenate([np.arange(o, o + n) for o, n in
                                    zip(coffs, spec["cused"] if cut else spec["clens"])])
            ck = spec["ckv"][crows]
            kw.update(k_cmp=ck, v_cmp=ck, cmp_lens=spec["cused"] if cut else spec["clens"],
                      cmp_idx=spec["cidx"][rows], cmp_ratio=spec["ratio"], ori_mask="band",
                      win_left=3, win_right=1)
            if not cut:
                kw["cmp_used"] = spec["cused"]
    return Problem(q=q, **kw), rows


@pytest.mark.parametrize("kind", ["token", "block", "swa_cmp"])
def test_used_lengths_equal_the_cut_problem(kind):
    spec = _spec(kind, seed={"token": 3, "block": 5, "swa_cmp": 7}[kind])
    pad, _ = _problem(spec, LENS, cut=False)
    cut, keep = _problem(spec, USED, cut=True)
    Op, lp = oracle.forward(pad, rounded=False)
    Oc, lc = oracle.forward(cut, rounded=False)
    np.testing.assert_allclose(Op[keep], Oc, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lp[keep], lc, rtol=1e-13, atol=1e-13)
    # rows past sequsedQ: O = 0 and lse = the sink alone
    drop = np.setdiff1d(np.arange(pad.T), keep)
    assert np.all(Op[drop] == 0)
    np.testing.assert_allclose(lp[drop], np.broadcast_to(spec["sinks"], lp[drop].shape), rtol=0, atol=0)
    rp = oracle.backward(pad, Op, lp, spec["do"], rounded=False)
    rc = oracle.backward(cut, Oc, lc, spec["do"][keep], rounded=False)
    np.testing.assert_allclose(rp["dq"][keep], rc["dq"], rtol=1e-12, atol=1e-12)
    assert np.all(rp["dq"][drop] == 0)
    np.testing.assert_allclose(rp["dsinks"], rc["dsinks"], rtol=1e-12, atol=1e-12)
    for key in [k for k in rp if k in ("dk", "dv", "dkv")]:
        np.testing.assert_allclose(rp[key][keep], rc[key], rtol=1e-12, atol=1e-12)
        assert np.all(rp[key][drop] == 0), key
    if "dcmp" in rp:
        coffs = np.cumsum((0,) + spec["clens"][:-1])
        ckeep = np.concatenate([np.arange(o, o + n) for o, n in zip(coffs, spec["cused"])])
        np.testing.assert_allclose(rp["dcmp"][ckeep], rc["dcmp"], rtol=1e-12, atol=1e-12)
        cdrop = np.setdiff1d(np.arange(rp["dcmp"].shape[0]), ckeep)
        assert np.all(rp["dcmp"][cdrop] == 0)


def test_full_used_lengths_change_nothing():
    spec = _spec("token", seed=11)
    a, _ = _problem(spec, LENS, cut=True)          # no used lengths
    kw = dict(q_used=LENS, kv_used=LENS)
    b = Problem(q=a.q, k_ori=a.k_ori, v_ori=a.v_ori, kv_shared=True, q_lens=LENS, kv_lens=LENS, Hq=a.Hq,
                Hkv=a.Hkv, d_qk=a.d_qk, d_v=a.d_v, scale=a.scale, ori_idx=a.ori_idx, sinks=a.sinks, **kw)
    Oa, la = oracle.forward(a, rounded=False)
    Ob, lb = oracle.forward(b, rounded=False)
    np.testing.assert_array_equal(Oa, Ob)
    np.testing.assert_array_equal(la, lb)
