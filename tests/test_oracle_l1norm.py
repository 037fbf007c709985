"""Pins for the oracle's SoftmaxL1Norm outputs (oriSoftmaxL1Norm / cmpSoftmaxL1Norm).

SparseFlashMlaGrad, "Parameter Description": two FLOAT32 outputs, the softmax
computed from the query and the original / compressed KV;
aclnnSparseLightningIndexerGradKLLoss, "Formula": the target distribution p is
the attention scores summed over all heads, then L1-normalised along the context.
Each test checks the oracle against something computed another way: a closed
form, a dense softmax over an explicit mask, or the sink's share of the softmax.
"""

import math

import numpy as np

import oracle
from oracle import Problem


def _token_problem(seed, Hkv=2, G=3, dup=False, zero_q=False, sinks=True, cmp=False):
    """Token-level selection over two sequences, distinct index lists per kv-head."""
    rng = np.random.default_rng(seed)
    lens, d, topk = (9, 6), 5, 4
    T, Hq = sum(lens), Hkv * G
    q = np.zeros((T, Hq, d)) if zero_q else rng.standard_normal((T, Hq, d))
    kv = rng.standard_normal((T, Hkv, d))
    idx = np.full((T, Hkv, topk), -1, dtype=np.int64)
    off = 0
    for L in lens:
        for t in range(L):
            for g in range(Hkv):
                sel = rng.permutation(L)[:rng.integers(0, topk + 1)]   # future rows too (masked)
                idx[off + t, g, :len(sel)] = sel
                idx[off + t, g] = rng.permutation(idx[off + t, g])     # -1 slots in between
        off += L
    if dup:
        idx[4, 0, :3] = [1, 1, 0]
    kw = {}
    if cmp:
        ratio, ctopk = 2, 3
        clens = tuple(L // ratio for L in lens)
        cidx = np.full((T, Hkv, ctopk), -1, dtype=np.int64)
        off = 0
        for L, C in zip(lens, clens):
            for t in range(L):
                for g in range(Hkv):
                    sel = rng.permutation(C)[:rng.integers(0, ctopk + 1)]
                    cidx[off + t, g, :len(sel)] = sel
            off += L
        ck = rng.standard_normal((sum(clens), Hkv, d))
        kw = dict(k_cmp=ck, v_cmp=ck, cmp_lens=clens, cmp_idx=cidx, cmp_ratio=ratio)
    s = rng.standard_normal(Hq) if sinks else None
    return Problem(q=q, k_ori=kv, v_ori=kv, kv_shared=True, q_lens=lens, kv_lens=lens, Hq=Hq, Hkv=Hkv,
                   d_qk=d, d_v=d, scale=0.6, block_size=1, ori_idx=idx, sinks=s, **kw), lens


def _block_problem(seed, zero_q=False):
    rng = np.random.default_rng(seed)
    lens, Hq, Hkv, d, bs, topk = (13, 9), 4, 2, 6, 4, 4
    T = sum(lens)
    q = np.zeros((T, Hq, d)) if zero_q else rng.standard_normal((T, Hq, d))
    k, v = rng.standard_normal((T, Hkv, d)), rng.standard_normal((T, Hkv, d))
    idx = np.full((T, Hkv, topk), -1, dtype=np.int64)
    off = 0
    for L in lens:
        nblk = (L + bs - 1) // bs
        for t in range(L):
            for g in range(Hkv):
                sel = rng.permutation(nblk)[:rng.integers(1, topk + 1)]
                idx[off + t, g, :len(sel)] = sel
        off += L
    olen = rng.integers(0, topk + 1, (T, Hkv))
    return Problem(q=q, k_ori=k, v_ori=v, kv_shared=False, q_lens=lens, kv_lens=lens, Hq=Hq, Hkv=Hkv,
                   d_qk=d, d_v=d, scale=0.7, block_size=bs, ori_idx=idx, ori_topk_len=olen,
                   sinks=rng.standard_normal(Hq)), lens, bs, idx, olen


def test_zero_query_gives_visible_row_shares():
    """q = 0 makes every score 0, so P is the same for every visible row of a head and
    the normalised output of slot s is (visible rows of s) / (visible rows of all slots),
    whatever the sinks and lse.  Visibility counted here by explicit loops."""
    p, lens, bs, idx, olen = _block_problem(7, zero_q=True)
    _, lse = oracle.forward(p, rounded=False)
    ori, cmp = oracle.softmax_l1norm(p, lse)
    assert cmp is None
    off = 0
    for L in lens:
        for t in range(L):
            for g in range(p.Hkv):
                counts = []
                for s in range(idx.shape[2]):
                    x = int(idx[off + t, g, s])
                    n = 0
                    if s < olen[off + t, g] and x >= 0:
                        for r in range(x * bs, x * bs + bs):
                            if r < L and r <= t:
                                n += 1
                    counts.append(n)
                tot = sum(counts)
                want = [c / tot if tot else 0.0 for c in counts]
                np.testing.assert_allclose(ori[off + t, g], want, atol=1e-13)
        off += L


def test_matches_a_dense_softmax_over_an_explicit_mask():
    """Dense scores for every head against every key of the sequence, a boolean mask
    built from the index lists, lse computed here from that mask (sink included), P
    summed over the heads of each kv-head at the selected keys, then normalised."""
    p, lens = _token_problem(11)
    _, lse_oracle = oracle.forward(p, rounded=False)
    ori, _ = oracle.softmax_l1norm(p, lse_oracle)
    off = 0
    for L in lens:
        for t in range(L):
            tq = off + t
            for g in range(p.Hkv):
                heads = range(g * p.G, (g + 1) * p.G)
                mask = np.zeros(L, dtype=bool)
                for x in p.ori_idx[tq, g]:
                    if x >= 0 and x <= t:
                        mask[x] = True
                acc = np.zeros(p.ori_idx.shape[2])
                for h in heads:
                    S = p.scale * (p.k_ori[off:off + L, g] @ p.q[tq, h])        # [L]
                    z = np.exp(S[mask]).sum() + math.exp(p.sinks[h])
                    P = np.exp(S - math.log(z))
                    for s, x in enumerate(p.ori_idx[tq, g]):
                        if x >= 0 and mask[x]:
                            acc[s] += P[x]
                want = acc / acc.sum() if acc.sum() > 0 else acc
                np.testing.assert_allclose(ori[tq, g], want, rtol=1e-12, atol=1e-14)
        off += L


def test_unnormalised_total_is_one_minus_the_sink_share():
    """Summed over every slot of both outputs, the unnormalised P of a head is the whole
    softmax minus the sink's share: sum_h (1 - exp(sink_h - lse_h)) per unit."""
    p, lens = _token_problem(13, cmp=True)
    _, lse = oracle.forward(p, rounded=False)
    for tq, g in p.all_units():
        hs = slice(g * p.G, (g + 1) * p.G)
        a_ori, a_cmp = oracle.unit_softmax_l1norm(p, tq, g, lse[tq, hs], normalize=False)
        want = float((1.0 - np.exp(p.sinks[hs] - lse[tq, hs])).sum())
        np.testing.assert_allclose(a_ori.sum() + a_cmp.sum(), want, rtol=1e-12, atol=1e-14)


def test_each_output_sums_to_one_and_empty_slots_are_zero():
    p, _ = _token_problem(17, cmp=True)
    _, lse = oracle.forward(p, rounded=False)
    ori, cmp = oracle.softmax_l1norm(p, lse)
    for out, idx in ((ori, p.ori_idx), (cmp, p.cmp_idx)):
        assert np.all(out >= 0)
        assert np.all(out[idx < 0] == 0)
        sums = out.sum(axis=2)
        assert np.all((np.abs(sums - 1) < 1e-12) | (sums == 0))
        assert np.any(sums == 1) or np.any(np.abs(sums - 1) < 1e-12)


def test_duplicate_slots_get_the_same_share():
    """A row named by two slots is gathered twice (multiplicity): both slots carry its P."""
    p, _ = _token_problem(19, Hkv=1, dup=True)
    _, lse = oracle.forward(p, rounded=False)
    ori, _ = oracle.softmax_l1norm(p, lse)
    assert ori[4, 0, 0] > 0
    np.testing.assert_allclose(ori[4, 0, 0], ori[4, 0, 1], rtol=1e-15)


def test_heads_of_other_kv_heads_do_not_mix():
    """Changing the queries of kv-head 1's heads leaves kv-head 0's output unchanged."""
    p, _ = _token_problem(23)
    _, lse = oracle.forward(p, rounded=False)
    ori0, _ = oracle.softmax_l1norm(p, lse)
    q2 = p.q.copy()
    q2[:, p.G:] = np.random.default_rng(1).standard_normal(q2[:, p.G:].shape)
    p2, _ = _token_problem(23)
    p2.q = q2
    _, lse2 = oracle.forward(p2, rounded=False)
    ori2, _ = oracle.softmax_l1norm(p2, lse2)
    np.testing.assert_array_equal(ori0[:, 0], ori2[:, 0])
    assert not np.allclose(ori0[:, 1], ori2[:, 1])
