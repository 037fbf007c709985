"""Pins for the paged KV cache in the oracle (aclnnNsaSelectedAttentionInfer: "paged
attention obtains the kvCache"; "Only paged attention is supported"; a few query
tokens per batch).

A cache of pages addressed through a block table must give what the same keys and
values give laid out contiguously per sequence, for block and token selection.
"""

import numpy as np
import pytest

import oracle
from oracle import Problem


def _paged_case(kind, seed):
    rng = np.random.default_rng(seed)
    B, s_q, Hq, Hkv, d, page = 3, 2, 4, 2, 6, 4
    kv_len = np.array([13, 7, 20])                      # actual KV tokens per sequence
    max_pages = int(np.ceil(kv_len.max() / page)) + 1
    n_pages = B * max_pages + 3
    perm = rng.permutation(n_pages)                     # physical pages in shuffled order
    table = perm[:B * max_pages].reshape(B, max_pages)
    kc = rng.standard_normal((n_pages * page, Hkv, d))
    vc = rng.standard_normal((n_pages * page, Hkv, d))
    q = rng.standard_normal((B * s_q, Hq, d))
    cap = max_pages * page
    if kind == "block":
        bs, topk = 4, 3
        idx = np.full((B * s_q, Hkv, topk), -1, dtype=np.int64)
        for b in range(B):
            for t in range(s_q):
                ta = t + kv_len[b] - s_q
                for g in range(Hkv):
                    sel = rng.permutation(ta // bs + 1)[:topk]
                    idx[b * s_q + t, g, :len(sel)] = sel
    else:
        bs, topk = 1, 5
        idx = np.full((B * s_q, Hkv, topk), -1, dtype=np.int64)
        for b in range(B):
            for t in range(s_q):
                ta = t + kv_len[b] - s_q
                for g in range(Hkv):
                    sel = rng.permutation(ta + 1)[:topk]
                    idx[b * s_q + t, g, :len(sel)] = sel
    sinks = rng.standard_normal(Hq)
    paged = Problem(q=q, k_ori=kc, v_ori=vc, kv_shared=False, q_lens=[s_q] * B, kv_lens=[cap] * B, Hq=Hq,
                    Hkv=Hkv, d_qk=d, d_v=d, scale=0.5, block_size=bs, ori_idx=idx, sinks=sinks,
                    kv_used=kv_len, block_table=table, page_size=page)
    # the same keys and values, contiguous per sequence
    rows = [table[b, np.arange(L) // page] * page + np.arange(L) % page for b, L in enumerate(kv_len)]
    k = np.concatenate([kc[r] for r in rows])
    v = np.concatenate([vc[r] for r in rows])
    flat = Problem(q=q, k_ori=k, v_ori=v, kv_shared=False, q_lens=[s_q] * B, kv_lens=list(kv_len), Hq=Hq,
                   Hkv=Hkv, d_qk=d, d_v=d, scale=0.5, block_size=bs, ori_idx=idx, sinks=sinks)
    return paged, flat


@pytest.mark.parametrize("kind", ["block", "token"])
def test_paged_cache_equals_contiguous_layout(kind):
    paged, flat = _paged_case(kind, seed={"block": 3, "token": 4}[kind])
    Op, lp = oracle.forward(paged, rounded=False)
    Of, lf = oracle.forward(flat, rounded=False)
    np.testing.assert_array_equal(Op, Of)
    np.testing.assert_array_equal(lp, lf)
    # every query sees at least one key (the selections are causal and non-empty)
    assert np.all(np.isfinite(lp))


def test_block_table_is_used():
    """Swapping two pages in the table (and their contents in the cache) changes nothing;
    swapping only the table entries changes the result."""
    paged, _ = _paged_case("token", seed=9)
    O0, _ = oracle.forward(paged, rounded=False)
    t2 = paged.block_table.copy()
    t2[0, 0], t2[0, 1] = t2[0, 1], t2[0, 0]
    bad = Problem(q=paged.q, k_ori=paged.k_ori, v_ori=paged.v_ori, kv_shared=False, q_lens=list(paged.q_len),
                  kv_lens=list(paged.kv_len), Hq=paged.Hq, Hkv=paged.Hkv, d_qk=paged.d_qk, d_v=paged.d_v,
                  scale=paged.scale, block_size=1, ori_idx=paged.ori_idx, sinks=paged.sinks,
                  kv_used=paged.kv_used, block_table=t2, page_size=paged.page_size)
    O1, _ = oracle.forward(bad, rounded=False)
    assert not np.allclose(O0[:2], O1[:2])
    kc, vc = paged.k_ori.copy(), paged.v_ori.copy()
    pa, pb, ps = paged.block_table[0, 0], paged.block_table[0, 1], paged.page_size
    for arr in (kc, vc):
        tmp = arr[pa * ps:(pa + 1) * ps].copy()
        arr[pa * ps:(pa + 1) * ps] = arr[pb * ps:(pb + 1) * ps]
        arr[pb * ps:(pb + 1) * ps] = tmp
    good = Problem(q=paged.q, k_ori=kc, v_ori=vc, kv_shared=False, q_lens=list(paged.q_len),
                   kv_lens=list(paged.kv_len), Hq=paged.Hq, Hkv=paged.Hkv, d_qk=paged.d_qk, d_v=paged.d_v,
                   scale=paged.scale, block_size=1, ori_idx=paged.ori_idx, sinks=paged.sinks,
                   kv_used=paged.kv_used, block_table=t2, page_size=paged.page_size)
    O2, _ = oracle.forward(good, rounded=False)
    np.testing.assert_array_equal(O0, O2)
