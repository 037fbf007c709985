"""Float64 CPU oracle for the lightning indexer's KL-loss backward.

TEST INFRASTRUCTURE ONLY.  The parity tests and the smoke check may import this
module; the CUDA product path never does.

aclnnSparseLightningIndexerGradKLLoss, "Formula":
  I[t, :]  = W[t, :] @ ReLU(q[t, :] @ K[:t, :]^T)      indexer scores of token t
  L        = sum_t KL(p[t, :] || Softmax(I[t, :]))      KL(a || b) = sum_i a_i log(a_i / b_i)
  dI[t, :] = Softmax(I[t, :]) - p[t, :]
  dW[t, :] = dI[t, :] @ ReLU(S[t, :])^T
  dq[t, :] = dS[t, :] @ K,   dK += dS[t, :]^T @ q[t, :]
with S = q K^T the raw scores and dS their gradient through ReLU and W:
dS[t, h, j] = dI[t, j] * W[t, h] * (S[t, h, j] > 0).

Readings taken where the page is silent or garbled:
  - the sparse operator scores only token t's selected keys (its topk index list,
    token indices local to its sequence); a slot is used when its index is >= 0, it
    lies before the row's topk length, and the key is not in t's future (the page's
    K[:t, :]); the softmax and the KL sum run over the used slots only;
  - "S is the result of the softmax operation on the QK matrix" is read as the raw
    scores q K^T, which ReLU(S) in the same formulas requires;
  - p is given per slot (the SoftmaxL1Norm outputs are of that shape); its entries
    at unused slots are ignored; 0 log 0 = 0;
  - no scale is applied to q K^T (the page prints none).
"""

from __future__ import annotations

import numpy as np

from .sparse_attn_ref import as_f64

__all__ = ["IndexerProblem", "indexer_slots", "unit_indexer_kl", "indexer_kl_grad"]


class IndexerProblem:
    """q [T, H, d], k [Tk, d] (one indexer key head), w [T, H], idx [T, topk] token
    indices (-1 = empty), p [T, topk] target distribution, optional topk_len [T];
    sequences by q_lens / kv_lens (token-major, packed)."""

    def __init__(self, *, q, k, w, idx, p, q_lens, kv_lens, topk_len=None):
        self.q, self.k = np.asarray(q), np.asarray(k)
        self.w = np.asarray(w, dtype=np.float64)
        self.idx = np.asarray(idx, dtype=np.int64)
        self.p = np.asarray(p, dtype=np.float64)
        self.topk_len = None if topk_len is None else np.asarray(topk_len, dtype=np.int64)
        self.q_len = np.asarray(q_lens, dtype=np.int64)
        self.kv_len = np.asarray(kv_lens, dtype=np.int64)
        self.q_start = np.concatenate([[0], np.cumsum(self.q_len)])[:-1]
        self.kv_start = np.concatenate([[0], np.cumsum(self.kv_len)])[:-1]
        self.T = int(self.q_len.sum())
        self.H, self.d = self.q.shape[1], self.q.shape[2]
        self._batch_of = np.repeat(np.arange(len(self.q_len)), self.q_len)


def indexer_slots(pr: IndexerProblem, tq: int) -> np.ndarray:
    """The used slots of token tq (positions in its index list), in slot order."""
    b = int(pr._batch_of[tq])
    t = tq - int(pr.q_start[b])
    ta = t + int(pr.kv_len[b]) - int(pr.q_len[b])
    n = pr.idx.shape[1] if pr.topk_len is None else max(0, min(pr.idx.shape[1], int(pr.topk_len[tq])))
    used = []
    for s in range(n):
        x = int(pr.idx[tq, s])
        if x < 0:
            continue
        if x >= int(pr.kv_len[b]):
            raise IndexError(f"indexer index out of range at token {tq}")
        if x <= ta:
            used.append(s)
    return np.asarray(used, dtype=np.int64)


def unit_indexer_kl(pr: IndexerProblem, tq: int) -> dict:
    """Loss and gradients of token tq: loss (scalar), dW [H], dq [H, d], and the key rows
    it touches with their dK contributions (rows [n] global, dK_rows [n, d])."""
    b = int(pr._batch_of[tq])
    slots = indexer_slots(pr, tq)
    q = as_f64(pr.q[tq])                                     # [H, d]
    out = dict(slots=slots, loss=0.0, dW=np.zeros(pr.H), dq=np.zeros((pr.H, pr.d)),
               rows=np.zeros(0, dtype=np.int64), dK_rows=np.zeros((0, pr.d)), I=np.zeros(0))
    if len(slots) == 0:
        return out
    rows = pr.kv_start[b] + pr.idx[tq, slots]
    K = as_f64(pr.k[rows])                                   # [n, d]
    S = q @ K.T                                              # [H, n] raw scores
    R = np.maximum(S, 0.0)
    I = pr.w[tq] @ R                                         # [n]
    m = I.max()
    e = np.exp(I - m)
    P = e / e.sum()                                          # Softmax(I)
    p = pr.p[tq, slots]
    dI = P - p
    with np.errstate(divide="ignore", invalid="ignore"):
        terms = np.where(p > 0, p * (np.log(p) - (I - m - np.log(e.sum()))), 0.0)
    dS = pr.w[tq][:, None] * (S > 0) * dI[None, :]           # [H, n]
    out.update(loss=float(terms.sum()), dW=R @ dI, dq=dS @ K, rows=rows, dK_rows=dS.T @ q, I=I)
    return out


def indexer_kl_grad(pr: IndexerProblem) -> dict:
    """Every token: loss [T], dq [T, H, d], dk [Tk, d], dw [T, H] (float64)."""
    loss = np.zeros(pr.T)
    dq = np.zeros((pr.T, pr.H, pr.d))
    dk = np.zeros((pr.k.shape[0], pr.d))
    dw = np.zeros((pr.T, pr.H))
    for tq in range(pr.T):
        r = unit_indexer_kl(pr, tq)
        loss[tq], dq[tq], dw[tq] = r["loss"], r["dq"], r["dW"]
        np.add.at(dk, r["rows"], r["dK_rows"])
    return dict(loss=loss, dq=dq, dk=dk, dw=dw)
