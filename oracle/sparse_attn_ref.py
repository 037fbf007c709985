"""Float64 CPU oracle for top-k index-selected sparse attention: forward and backward.

TEST INFRASTRUCTURE ONLY.  The parity tests, the smoke check and the CPU-baseline
leg of the benchmark may import this module; the CUDA product path never does,
and this module imports nothing from it.

What it computes is the plain definition, one query token at a time, in float64
(NumPy matmul as the only library step):

* Selection.  aclnnSparseFlashAttentionGrad, "Formula": selectedKey/selectedValue
  = Gather(key/value, topkIndices[i]) for 0 <= i < selectBlockCount, each index
  naming a block of contiguous rows.  SparseFlashMlaGrad, "Computation formula",
  Stage 1: cmp_ratio = 1 (SWA) selects the original KV, cmp_ratio = 4 (SCFA)
  concatenates the original KV with Gather(cmpKv, topkIndices[i]), any other
  ratio (CFA) concatenates the original KV with all of cmpKv; the
  "Parameter Description" table adds oriSparseIndices (token rows of the
  original KV), oriTopkLength / cmpTopkLength (usable slots per query row),
  oriMaskMode / cmpMaskMode and oriWinLeft / oriWinRight.
* Forward.  aclnnNsaSelectedAttentionInfer, "Formula":
  Softmax(query . key_topk^T / sqrt(d)) . value_topk, with the scale attribute
  (scaleValue) in place of 1/sqrt(d), an optional per-head sink logit in the
  softmax denominator, and lse = log of that denominator (natural log).
* Backward.  SparseFlashMlaGrad, "Computation formula", Stages 2-3, and
  aclnnSparseFlashAttentionGrad, "Formula", Phases 1-3:
      P  = SimpleSoftmax(Mask(Q selKv^T scale), lse) = exp(S - lse)
      dP = dO V^T
      dS = P o (dP - rowsum(dO o O))          (o = elementwise product)
      dQ = dS K scale,  dK = dS^T Q scale,  dV = P^T dO  (dKV = dK + dV if K = V)
      dSinks = sum over rows of -P_sink * sum_j P_j dP_j,  P_sink = exp(sink - lse)
* SoftmaxL1Norm outputs.  SparseFlashMlaGrad, "Parameter Description"
  (oriSoftmaxL1NormOptional / cmpSoftmaxL1NormOptional) with the target
  distribution of aclnnSparseLightningIndexerGradKLLoss, "Formula": P summed over
  the heads of a kv-head and over each slot's visible rows, L1-normalised along
  that output's slots.

Readings taken where the pages are silent or garbled (each is listed with its
reason in the design notes of this repository):
  - the "@" inside the dS formula of aclnnSparseFlashAttentionGrad is the
    elementwise product (SparseFlashMlaGrad prints "x");
  - block x covers rows [x*bs, (x+1)*bs) of the same sequence, rows past the
    sequence end are dropped;
  - an index < 0, or a slot at or past the row's topk length, selects nothing;
  - causal masks align the last query with the last key (bottom-right); the
    band mask keeps rows in [t - winLeft, t + winRight]; a compressed row c is
    visible when its last source token, (c + 1) * cmp_ratio - 1, is <= t;
  - duplicates in a row's index list are gathered with multiplicity;
  - a row with no visible key and no sink has lse = +inf and O = 0, and gives
    zero gradients;
  - with K = V, V is the first d_v columns of the shared KV row;
  - TND indices are positions local to their own sequence, like BSND;
  - sequsedQ / sequsedOriKv / sequsedCmpKv shorten each sequence to the tokens
    that take part: the effective lengths set the causal alignment and the
    sequence end; a query row past sequsedQ selects nothing (an empty row);
  - a paged KV cache maps logical row r of sequence b to physical row
    block_table[b, r // page_size] * page_size + r % page_size;
  - the compressed rows are gathered through cmp indices when there are any
    (SCFA); a compressed KV without indices contributes all its rows (CFA);
  - each SoftmaxL1Norm output is normalised over its own slots (ori and cmp
    separately), the sink is no slot, and an output exists only where its index
    list does.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "widen_bf16",
    "round_to_bf16_bits",
    "Problem",
    "visible_rows",
    "unit_forward",
    "unit_backward",
    "forward",
    "backward",
    "unit_softmax_l1norm",
    "softmax_l1norm",
    "unit_flops",
]


# ----------------------------------------------------------------------------
# bfloat16 <-> float64 (the oracle's own conversions)
# ----------------------------------------------------------------------------

def widen_bf16(u16: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float64, exactly (a bf16 is the top half of a binary32)."""
    u = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> bfloat16 bit patterns, round to nearest, ties to even, in one step.

    A bfloat16 keeps 8 significant bits, so for |x| in [2^(e-1), 2^e) its spacing
    is 2^(e-8) (never below 2^-133, the subnormal spacing).  Dividing by that
    power of two is exact, np.rint rounds half to even, and the result is exactly
    representable in binary32, whose top 16 bits are the bfloat16.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    spacing = np.ldexp(1.0, np.maximum(e - 8, -133))
    q = np.rint(x / spacing) * spacing
    q = np.where(np.isfinite(x), q, x)
    bits = q.astype(np.float32).view(np.uint32) >> np.uint32(16)
    return bits.astype(np.uint16)


def as_f64(x) -> np.ndarray:
    """float64 view of an array slice: bf16 bit patterns (uint16) are widened exactly."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return widen_bf16(x)
    return x.astype(np.float64, copy=False)


# ----------------------------------------------------------------------------
# Problem description
# ----------------------------------------------------------------------------

class Problem:
    """All inputs of one sparse-attention call, token-major.

    Tensors may be float64 or bf16 bit patterns (uint16); the latter are
    widened exactly to float64 row by row when a unit reads them.

    Arrays (T = total query tokens, Tk = total original KV rows, Tc = total
    compressed KV rows):
      q      [T, Hq, d_qk]
      k_ori  [Tk, Hkv, d_qk],  v_ori [Tk, Hkv, d_v]   (K = V: v_ori is k_ori[..., :d_v])
      k_cmp  [Tc, Hkv, d_qk],  v_cmp [Tc, Hkv, d_v]   (compressed KV, always K = V)
      ori_idx [T, Hkv, topk] int, cmp_idx [T, Hkv, cmp_topk] int (or None)
      ori_topk_len / cmp_topk_len [T, Hkv] int (or None)
      sinks [Hq] (or None)
    Sequences: q_start/q_len, kv_start/kv_len, cmp_start/cmp_len per batch.
    """

    def __init__(self, *, q, k_ori, v_ori, kv_shared, q_lens, kv_lens, Hq, Hkv,
                 d_qk, d_v, scale, block_size=1, ori_idx=None, ori_topk_len=None,
                 k_cmp=None, v_cmp=None, cmp_lens=None, cmp_idx=None,
                 cmp_topk_len=None, cmp_ratio=1, ori_mask="causal",
                 cmp_mask="causal", win_left=0, win_right=0, sinks=None,
                 q_used=None, kv_used=None, cmp_used=None, block_table=None, page_size=0):
        self.q = np.asarray(q)
        self.k_ori = np.asarray(k_ori)
        self.v_ori = np.asarray(v_ori)
        self.kv_shared = bool(kv_shared)
        self.Hq, self.Hkv, self.d_qk, self.d_v = Hq, Hkv, d_qk, d_v
        assert Hq % Hkv == 0
        self.G = Hq // Hkv
        self.scale = float(scale)
        self.block_size = int(block_size)
        self.ori_idx = None if ori_idx is None else np.asarray(ori_idx, dtype=np.int64)
        self.ori_topk_len = None if ori_topk_len is None else np.asarray(ori_topk_len, dtype=np.int64)
        self.k_cmp = None if k_cmp is None else np.asarray(k_cmp)
        self.v_cmp = None if v_cmp is None else np.asarray(v_cmp)
        self.cmp_idx = None if cmp_idx is None else np.asarray(cmp_idx, dtype=np.int64)
        self.cmp_topk_len = None if cmp_topk_len is None else np.asarray(cmp_topk_len, dtype=np.int64)
        self.cmp_ratio = int(cmp_ratio)
        self.ori_mask, self.cmp_mask = ori_mask, cmp_mask
        self.win_left, self.win_right = int(win_left), int(win_right)
        self.sinks = None if sinks is None else np.asarray(sinks, dtype=np.float64)
        self.q_len = np.asarray(q_lens, dtype=np.int64)
        self.kv_len = np.asarray(kv_lens, dtype=np.int64)
        self.q_start = np.concatenate([[0], np.cumsum(self.q_len)])[:-1]
        self.kv_start = np.concatenate([[0], np.cumsum(self.kv_len)])[:-1]
        if cmp_lens is None:
            cmp_lens = np.zeros_like(self.q_len)
        self.cmp_len = np.asarray(cmp_lens, dtype=np.int64)
        self.cmp_start = np.concatenate([[0], np.cumsum(self.cmp_len)])[:-1]
        self.T = int(self.q_len.sum())
        # sequsedQ / sequsedOriKv / sequsedCmpKv: tokens of each sequence that take part
        nb = len(self.q_len)
        self.q_used = self.q_len.copy() if q_used is None else np.minimum(self.q_len, np.asarray(q_used))
        self.kv_used = self.kv_len.copy() if kv_used is None else np.minimum(self.kv_len, np.asarray(kv_used))
        self.cmp_used = self.cmp_len.copy() if cmp_used is None else np.minimum(self.cmp_len, np.asarray(cmp_used))
        assert len(self.q_used) == len(self.kv_used) == len(self.cmp_used) == nb
        # paged KV cache (aclnnNsaSelectedAttentionInfer: "paged attention obtains the
        # kvCache"): k_ori / v_ori are the cache, [pages * page_size, Hkv, d]; logical row r
        # of sequence b lives in physical page block_table[b, r // page_size]
        self.block_table = None if block_table is None else np.asarray(block_table, dtype=np.int64)
        self.page_size = int(page_size)
        self._batch_of = np.repeat(np.arange(len(self.q_len)), self.q_len)
        assert self.q.shape == (self.T, Hq, d_qk)

    @property
    def Tk(self) -> int:
        return int(self.k_ori.shape[0])

    @property
    def Tc(self) -> int:
        return 0 if self.k_cmp is None else int(self.k_cmp.shape[0])

    def all_units(self):
        return [(tq, g) for tq in range(self.T) for g in range(self.Hkv)]

    @property
    def has_cmp(self) -> bool:
        return self.k_cmp is not None

    def batch_of(self, tq: int) -> int:
        return int(self._batch_of[tq])

    @classmethod
    def from_inputs(cls, w, inp: dict) -> "Problem":
        """Build from a workload description and the generator's arrays (bf16 as uint16,
        kept as bit patterns and widened when read)."""
        T = w.T
        q = inp["q"].reshape(T, w.Hq, w.d_qk)
        if w.kv_shared:
            kv = inp["kv"].reshape(T, w.Hkv, w.d_qk)
            k_ori, v_ori = kv, kv[..., :w.d_v]
        else:
            k_ori = inp["k"].reshape(T, w.Hkv, w.d_qk)
            v_ori = inp["v"].reshape(T, w.Hkv, w.d_v)
        lens = list(w.seq_lengths)
        kw = {}
        if "ori_idx" in inp:
            kw["ori_idx"] = inp["ori_idx"].reshape(T, w.Hkv, -1)
        if "ori_topk_len" in inp:
            kw["ori_topk_len"] = inp["ori_topk_len"].reshape(T, w.Hkv)
        if "cmp_kv" in inp:
            ck = inp["cmp_kv"].reshape(-1, w.Hkv, w.d_qk)
            kw.update(k_cmp=ck, v_cmp=ck[..., :w.d_v],
                      cmp_lens=np.diff(inp["cu_seqlens_cmp"]))
            if "cmp_idx" in inp:
                kw["cmp_idx"] = inp["cmp_idx"].reshape(T, w.Hkv, -1)
            if "cmp_topk_len" in inp:
                kw["cmp_topk_len"] = inp["cmp_topk_len"].reshape(T, w.Hkv)
        if "sinks" in inp:
            kw["sinks"] = inp["sinks"].astype(np.float64)
        for key, arg in (("seqused_q", "q_used"), ("seqused_kv", "kv_used"), ("seqused_cmp", "cmp_used")):
            if key in inp:
                kw[arg] = inp[key].astype(np.int64)
        return cls(q=q, k_ori=k_ori, v_ori=v_ori, kv_shared=w.kv_shared, q_lens=lens,
                   kv_lens=lens, Hq=w.Hq, Hkv=w.Hkv, d_qk=w.d_qk, d_v=w.d_v,
                   scale=w.scale, block_size=w.block_size, cmp_ratio=w.cmp_ratio,
                   ori_mask=w.ori_mask, cmp_mask=w.cmp_mask, win_left=w.win_left,
                   win_right=w.win_right, **kw)


# ----------------------------------------------------------------------------
# Selection (Stage 1 / the Gather formula) and masks
# ----------------------------------------------------------------------------

def visible_rows(p: Problem, tq: int, g: int):
    """Visible KV rows of query token ``tq`` (global) under kv-head ``g``.

    Returns (ori_rows, cmp_rows): int64 arrays of row numbers local to the
    token's sequence, in slot order (duplicates kept).
    """
    b = p.batch_of(tq)
    t = tq - int(p.q_start[b])
    Lk = int(p.kv_used[b])                    # the rows that take part (sequsedOriKv)
    ta = t + (Lk - int(p.q_used[b]))          # query position on the key axis
    if t >= int(p.q_used[b]):                 # past sequsedQ: the row selects nothing
        return np.zeros(0, dtype=np.int64), np.zeros(0, dtype=np.int64)

    # original KV: gathered through the ori indices, else all of it (SWA / SCFA / CFA)
    if p.ori_idx is not None:
        n = p.ori_idx.shape[2]
        if p.ori_topk_len is not None:
            n = max(0, min(n, int(p.ori_topk_len[tq, g])))
        idx = p.ori_idx[tq, g, :n]
        idx = idx[idx >= 0]
        bs = p.block_size
        if np.any(idx * bs >= Lk):
            raise IndexError(f"ori index out of range at token {tq}, kv-head {g}")
        ori = (idx[:, None] * bs + np.arange(bs)[None, :]).reshape(-1)
        ori = ori[ori < Lk]
    else:
        ori = np.arange(Lk, dtype=np.int64)
    if p.ori_mask == "causal":
        ori = ori[ori <= ta]
    elif p.ori_mask == "band":
        ori = ori[(ori >= ta - p.win_left) & (ori <= ta + p.win_right)]
    elif p.ori_mask != "none":
        raise ValueError(p.ori_mask)

    # compressed KV: gathered through the cmp indices (SCFA)
    cmp = np.zeros(0, dtype=np.int64)
    if p.has_cmp and p.cmp_idx is not None:
        n = p.cmp_idx.shape[2]
        if p.cmp_topk_len is not None:
            n = max(0, min(n, int(p.cmp_topk_len[tq, g])))
        c = p.cmp_idx[tq, g, :n]
        c = c[c >= 0]
        if np.any(c >= int(p.cmp_used[b])):
            raise IndexError(f"cmp index out of range at token {tq}, kv-head {g}")
        if p.cmp_mask == "causal":
            c = c[(c + 1) * p.cmp_ratio - 1 <= ta]
        elif p.cmp_mask != "none":
            raise ValueError(p.cmp_mask)
        cmp = c
    elif p.has_cmp:
        # CFA (Stage 1, the "else" case): every compressed row of the sequence
        c = np.arange(int(p.cmp_used[b]), dtype=np.int64)
        if p.cmp_mask == "causal":
            c = c[(c + 1) * p.cmp_ratio - 1 <= ta]
        elif p.cmp_mask != "none":
            raise ValueError(p.cmp_mask)
        cmp = c
    return ori, cmp


def kv_rows(p: Problem, b: int, rows) -> np.ndarray:
    """Storage rows of sequence b's (sequence-local) original-KV rows: contiguous from
    kv_start[b], or through the block table of a paged cache."""
    rows = np.asarray(rows, dtype=np.int64)
    if p.block_table is None:
        return p.kv_start[b] + rows
    return p.block_table[b, rows // p.page_size] * p.page_size + rows % p.page_size


def _gather(p: Problem, tq: int, g: int):
    b = p.batch_of(tq)
    ori, cmp = visible_rows(p, tq, g)
    K = as_f64(p.k_ori[kv_rows(p, b, ori), g])
    V = as_f64(p.v_ori[kv_rows(p, b, ori), g])
    if len(cmp):
        K = np.concatenate([K, as_f64(p.k_cmp[p.cmp_start[b] + cmp, g])])
        V = np.concatenate([V, as_f64(p.v_cmp[p.cmp_start[b] + cmp, g])])
    return ori, cmp, K, V


# ----------------------------------------------------------------------------
# Forward (selected attention with optional sinks)
# ----------------------------------------------------------------------------

def unit_forward(p: Problem, tq: int, g: int):
    """O [G, d_v] and lse [G] (float64) for the G query heads of kv-head g at token tq."""
    hs = slice(g * p.G, (g + 1) * p.G)
    Q = as_f64(p.q[tq, hs])
    _, _, K, V = _gather(p, tq, g)
    S = p.scale * (Q @ K.T)                               # [G, n] scaled scores
    sink = None if p.sinks is None else p.sinks[hs]
    if K.shape[0] == 0 and sink is None:
        return np.zeros((p.G, p.d_v)), np.full(p.G, np.inf)
    m = np.full(p.G, -np.inf)
    if K.shape[0]:
        m = S.max(axis=1)
    if sink is not None:
        m = np.maximum(m, sink)
    Z = np.exp(S - m[:, None]).sum(axis=1)
    if sink is not None:
        Z = Z + np.exp(sink - m)
    lse = m + np.log(Z)
    P = np.exp(S - lse[:, None])
    return P @ V, lse


def forward(p: Problem, units=None, rounded: bool = True):
    """Forward over every unit (token, kv-head), or over ``units`` only.

    With ``units=None`` returns (O, lse): O [T, Hq, d_v], lse [T, Hq].  With a
    list of units returns a dict {(tq, g): (O [G, d_v], lse [G])}.  Rounded: O
    as bf16 bits and lse as float32; otherwise float64.
    """
    def fin(o, l):
        return (round_to_bf16_bits(o), l.astype(np.float32)) if rounded else (o, l)

    if units is not None:
        return {(tq, g): fin(*unit_forward(p, tq, g)) for tq, g in units}
    O = np.zeros((p.T, p.Hq, p.d_v))
    lse = np.zeros((p.T, p.Hq))
    for tq, g in p.all_units():
        o, l = unit_forward(p, tq, g)
        O[tq, g * p.G:(g + 1) * p.G] = o
        lse[tq, g * p.G:(g + 1) * p.G] = l
    return fin(O, lse)


# ----------------------------------------------------------------------------
# Backward (Stages 2-3 / Phases 1-3)
# ----------------------------------------------------------------------------

def unit_backward(p: Problem, tq: int, g: int, O, lse, dO):
    """Everything the backward derives for one unit.

    ``O`` [G, d_v], ``lse`` [G], ``dO`` [G, d_v] are the float64 inputs of this
    unit.  Returns a dict with ori/cmp rows, S, P, dP, Delta, dS, dQ [G, d_qk],
    dK_rows [n, d_qk], dV_rows [n, d_v], P_sink [G] and dSinks [G].
    """
    hs = slice(g * p.G, (g + 1) * p.G)
    Q = as_f64(p.q[tq, hs])
    ori, cmp, K, V = _gather(p, tq, g)
    S = p.scale * (Q @ K.T)
    P = np.exp(S - lse[:, None])                          # SimpleSoftmax(S, lse)
    dP = dO @ V.T
    Delta = (dO * O).sum(axis=1)                          # rowsum(dO o O)
    dS = P * (dP - Delta[:, None])
    out = dict(ori=ori, cmp=cmp, S=S, P=P, dP=dP, Delta=Delta, dS=dS,
               dQ=p.scale * (dS @ K),
               dK_rows=p.scale * (dS.T @ Q),
               dV_rows=P.T @ dO)
    if p.sinks is not None:
        psink = np.exp(p.sinks[hs] - lse)
        out["P_sink"] = psink
        out["dSinks"] = -psink * (P * dP).sum(axis=1)
    return out


def _scatter_add(dst, rows, vals):
    """dst[rows] += vals, adding repeated rows once per occurrence."""
    if len(np.unique(rows)) == len(rows):
        dst[rows] += vals
    else:
        np.add.at(dst, rows, vals)


def backward(p: Problem, O, lse, dO, units=None, rounded: bool = True):
    """Backward over every unit, or over ``units`` only (then dK/dV are partial sums).

    ``O``, ``dO`` [T, Hq, d_v] and ``lse`` [T, Hq]: float64 arrays, or bf16 bit
    patterns / float32 (widened exactly when read).  Returns a dict: dq
    [T, Hq, d_qk] (a dict {(tq, g): [G, d_qk]} when ``units`` is given); dk
    [Tk, Hkv, d_qk] and dv [Tk, Hkv, d_v], or dkv [Tk, Hkv, d_qk] when K = V;
    dcmp [Tc, Hkv, d_qk] when there is a compressed KV; dsinks [Hq] when there
    are sinks.  Rounded: bf16 bits for every tensor but dsinks (float32);
    otherwise float64.
    """
    dk = np.zeros((p.Tk, p.Hkv, p.d_qk))
    dv = np.zeros((p.Tk, p.Hkv, p.d_v))
    dkc = np.zeros((p.Tc, p.Hkv, p.d_qk))
    dvc = np.zeros((p.Tc, p.Hkv, p.d_v))
    dsinks = np.zeros(p.Hq)
    if units is None:
        dq = np.zeros((p.T, p.Hq, p.d_qk))
        todo = p.all_units()
    else:
        dq = {}
        todo = units
    for tq, g in todo:
        hs = slice(g * p.G, (g + 1) * p.G)
        r = unit_backward(p, tq, g, as_f64(O[tq, hs]), as_f64(lse[tq, hs]), as_f64(dO[tq, hs]))
        if units is None:
            dq[tq, hs] = r["dQ"]
        else:
            dq[(tq, g)] = r["dQ"]
        b = p.batch_of(tq)
        no = len(r["ori"])
        _scatter_add(dk[:, g], kv_rows(p, b, r["ori"]), r["dK_rows"][:no])
        _scatter_add(dv[:, g], kv_rows(p, b, r["ori"]), r["dV_rows"][:no])
        if len(r["cmp"]):
            _scatter_add(dkc[:, g], p.cmp_start[b] + r["cmp"], r["dK_rows"][no:])
            _scatter_add(dvc[:, g], p.cmp_start[b] + r["cmp"], r["dV_rows"][no:])
        if p.sinks is not None:
            dsinks[hs] += r["dSinks"]
    res = {"dq": dq}
    if p.kv_shared:
        dkv = dk.copy()
        dkv[..., :p.d_v] += dv
        res["dkv"] = dkv
    else:
        res["dk"], res["dv"] = dk, dv
    if p.k_cmp is not None:
        dc = dkc.copy()
        dc[..., :p.d_v] += dvc
        res["dcmp"] = dc
    if p.sinks is not None:
        res["dsinks"] = dsinks
    if rounded:
        for key in list(res):
            if key == "dsinks":
                res[key] = res[key].astype(np.float32)
            elif key == "dq" and units is not None:
                res[key] = {u: round_to_bf16_bits(v) for u, v in res[key].items()}
            else:
                res[key] = round_to_bf16_bits(res[key])
    return res


# ----------------------------------------------------------------------------
# The SoftmaxL1Norm outputs (the indexer loss's target distribution)
# ----------------------------------------------------------------------------

def _slot_rows(p: Problem, tq: int, g: int, kind: str):
    """For each ori (kind "ori") or cmp slot of unit (tq, g): the rows it selects that
    survive the masks (sequence-local, possibly empty), by the same rules as
    visible_rows, slot by slot."""
    b = p.batch_of(tq)
    t = tq - int(p.q_start[b])
    Lk = int(p.kv_used[b])
    ta = t + (Lk - int(p.q_used[b]))
    idx_all = p.ori_idx if kind == "ori" else p.cmp_idx
    if t >= int(p.q_used[b]):                 # past sequsedQ: every slot is empty
        return [np.zeros(0, dtype=np.int64) for _ in range(idx_all.shape[2])]
    out = []
    if kind == "ori":
        n_all = p.ori_idx.shape[2]
        n = n_all if p.ori_topk_len is None else max(0, min(n_all, int(p.ori_topk_len[tq, g])))
        bs = p.block_size
        for s in range(n_all):
            x = int(p.ori_idx[tq, g, s])
            if s >= n or x < 0:
                out.append(np.zeros(0, dtype=np.int64))
                continue
            if x * bs >= Lk:
                raise IndexError(f"ori index out of range at token {tq}, kv-head {g}")
            rows = x * bs + np.arange(bs)
            rows = rows[rows < Lk]
            if p.ori_mask == "causal":
                rows = rows[rows <= ta]
            elif p.ori_mask == "band":
                rows = rows[(rows >= ta - p.win_left) & (rows <= ta + p.win_right)]
            out.append(rows)
    else:
        n_all = p.cmp_idx.shape[2]
        n = n_all if p.cmp_topk_len is None else max(0, min(n_all, int(p.cmp_topk_len[tq, g])))
        for s in range(n_all):
            c = int(p.cmp_idx[tq, g, s])
            if s >= n or c < 0:
                out.append(np.zeros(0, dtype=np.int64))
                continue
            if c >= int(p.cmp_used[b]):
                raise IndexError(f"cmp index out of range at token {tq}, kv-head {g}")
            ok = p.cmp_mask != "causal" or (c + 1) * p.cmp_ratio - 1 <= ta
            out.append(np.array([c] if ok else [], dtype=np.int64))
    return out


def unit_softmax_l1norm(p: Problem, tq: int, g: int, lse, normalize: bool = True):
    """oriSoftmaxL1Norm / cmpSoftmaxL1Norm of query token tq under kv-head g.

    SparseFlashMlaGrad, "Parameter Description": two FLOAT32 outputs, the softmax
    result computed from the query and the original (resp. compressed) KV.
    aclnnSparseLightningIndexerGradKLLoss, "Formula": the indexer's target
    distribution p is the main attention scores summed over all heads, then
    L1-normalised along the context.  Here P = exp(scale q.k - lse) is the
    backward's recomputed softmax (``lse`` [G] of this unit, sink included; the
    sink is no context position).  Entry s of an output sums P over the G heads of
    kv-head g and over the visible rows its slot selects; each output is then
    divided by its own sum (all zeros when that sum is 0).

    Returns (ori [topk] or None, cmp [cmp_topk] or None), float64; None where the
    problem has no index list of that kind.
    """
    hs = slice(g * p.G, (g + 1) * p.G)
    Q = as_f64(p.q[tq, hs])
    lse = np.asarray(lse, dtype=np.float64)
    b = p.batch_of(tq)
    res = []
    for kind in ("ori", "cmp"):
        if (kind == "ori" and p.ori_idx is None) or (kind == "cmp" and (p.cmp_idx is None or not p.has_cmp)):
            res.append(None)
            continue
        slots = _slot_rows(p, tq, g, kind)
        a = np.zeros(len(slots))
        for s, rows in enumerate(slots):
            if len(rows) == 0:
                continue
            if kind == "ori":
                K = as_f64(p.k_ori[kv_rows(p, b, rows), g])
            else:
                K = as_f64(p.k_cmp[p.cmp_start[b] + rows, g])
            P = np.exp(p.scale * (Q @ K.T) - lse[:, None])   # [G, rows of the slot]
            a[s] = P.sum()
        if normalize:
            tot = a.sum()
            a = a / tot if tot > 0 else np.zeros_like(a)
        res.append(a)
    return tuple(res)


def softmax_l1norm(p: Problem, lse, units=None):
    """Both outputs over every unit: (ori [T, Hkv, topk] or None, cmp [T, Hkv, cmp_topk]
    or None), float64, from ``lse`` [T, Hq] (float32 or float64).  With ``units`` only
    those units are filled (the rest stay zero)."""
    ori = None if p.ori_idx is None else np.zeros((p.T, p.Hkv, p.ori_idx.shape[2]))
    cmp = None if (p.cmp_idx is None or not p.has_cmp) else np.zeros((p.T, p.Hkv, p.cmp_idx.shape[2]))
    for tq, g in (p.all_units() if units is None else units):
        hs = slice(g * p.G, (g + 1) * p.G)
        o, c = unit_softmax_l1norm(p, tq, g, np.asarray(lse, dtype=np.float64)[tq, hs])
        if ori is not None:
            ori[tq, g] = o
        if cmp is not None:
            cmp[tq, g] = c
    return ori, cmp


def unit_flops(p: Problem, tq: int, g: int) -> tuple:
    """(forward, backward) FLOPs of one unit counted over visible (row, head, key) triples."""
    ori, cmp = visible_rows(p, tq, g)
    n = (len(ori) + len(cmp)) * p.G
    return 2 * (p.d_qk + p.d_v) * n, 2 * (3 * p.d_qk + 2 * p.d_v) * n

