"""Pins for the oracle's lightning-indexer KL-loss backward
(aclnnSparseLightningIndexerGradKLLoss, "Formula").  Each checks the oracle against
something computed another way: central finite differences of the loss it reports,
the fixed point p = Softmax(I), the sign of a KL divergence, and the slots it must
ignore."""

import numpy as np

from oracle.indexer_ref import IndexerProblem, indexer_kl_grad, indexer_slots, unit_indexer_kl


def _problem(seed, H=3, d=4, topk=5, lens=(7, 5)):
    rng = np.random.default_rng(seed)
    T = sum(lens)
    q = rng.standard_normal((T, H, d))
    k = rng.standard_normal((T, d))
    w = rng.standard_normal((T, H))
    idx = np.full((T, topk), -1, dtype=np.int64)
    off = 0
    for L in lens:
        for t in range(L):
            sel = rng.permutation(L)[:rng.integers(1, topk + 1)]   # future keys too (unused)
            idx[off + t, :len(sel)] = sel
            idx[off + t] = rng.permutation(idx[off + t])          # -1 slots in between
        off += L
    p = rng.random((T, topk))
    pr = IndexerProblem(q=q, k=k, w=w, idx=idx, p=p, q_lens=lens, kv_lens=lens,
                        topk_len=rng.integers(1, topk + 1, T))
    # the target: a distribution over each token's used slots
    for tq in range(T):
        s = indexer_slots(pr, tq)
        if len(s):
            pr.p[tq, s] /= pr.p[tq, s].sum()
    return pr


def _total_loss(pr):
    return indexer_kl_grad(pr)["loss"].sum()


def test_gradients_match_finite_differences():
    pr = _problem(3)
    g = indexer_kl_grad(pr)
    eps = 1e-6
    for name, arr, grad in (("q", pr.q, g["dq"]), ("k", pr.k, g["dk"]), ("w", pr.w, g["dw"])):
        num = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = arr[i]
            arr[i] = old + eps
            lp = _total_loss(pr)
            arr[i] = old - eps
            lm = _total_loss(pr)
            arr[i] = old
            num[i] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-5, atol=1e-7, err_msg=name)


def test_target_equal_to_the_indexer_softmax_gives_zero():
    pr = _problem(5)
    for tq in range(pr.T):
        r = unit_indexer_kl(pr, tq)
        if len(r["slots"]):
            e = np.exp(r["I"] - r["I"].max())
            pr.p[tq, r["slots"]] = e / e.sum()
    g = indexer_kl_grad(pr)
    np.testing.assert_allclose(g["loss"], 0.0, atol=1e-12)
    for key in ("dq", "dk", "dw"):
        np.testing.assert_allclose(g[key], 0.0, atol=1e-12)


def test_kl_is_non_negative_and_unused_slots_are_ignored():
    pr = _problem(7)
    g = indexer_kl_grad(pr)
    assert np.all(g["loss"] >= -1e-12)
    used = np.zeros_like(pr.p, dtype=bool)
    for tq in range(pr.T):
        used[tq, indexer_slots(pr, tq)] = True
    pr.p[~used] = 123.0                                       # never read
    g2 = indexer_kl_grad(pr)
    for key in g:
        np.testing.assert_array_equal(g[key], g2[key])
    assert (~used).any() and used.any()


def test_a_single_used_slot():
    """One used slot: Softmax(I) = 1, so dI = 1 - p there and the loss is -p log p... with
    p = 1 everything vanishes."""
    pr = _problem(9)
    tq = 3
    s = indexer_slots(pr, tq)
    pr.topk_len[tq] = s[0] + 1 if len(s) else 0
    r = unit_indexer_kl(pr, tq)
    if len(r["slots"]) == 1:
        pr.p[tq, r["slots"][0]] = 1.0
        r = unit_indexer_kl(pr, tq)
        assert r["loss"] == 0.0
        assert np.all(r["dq"] == 0) and np.all(r["dW"] == 0)
