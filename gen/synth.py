"""Seeded input generation for the sparse-attention workloads.

One ``numpy.random.Generator(PCG64(seed))`` stream per workload, drawn in a
fixed order: q, k / kv, v, dO, sinks, index sets, topk lengths.  Normal values
are drawn in float32 and rounded to bfloat16 (round to nearest, ties to even);
bfloat16 tensors are carried as their raw uint16 bit patterns.

Nothing here computes attention: the only arithmetic is drawing numbers,
rounding them to bfloat16 and the mean-pooling that stands in for the upstream
KV compressor (whose algorithm the pages do not give).
"""

from __future__ import annotations

import numpy as np

from .configs import Workload

_CHUNK = 1 << 24


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (RNE); return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def f32_from_bf16_bits(u: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape, mul: float = 1.0) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        x = rng.standard_normal(hi - lo, dtype=np.float32)
        if mul != 1.0:
            x *= np.float32(mul)
        out[lo:hi] = bf16_bits_from_f32(x)
    return out.reshape(shape)


def _smallest_k(keys: np.ndarray, k: int) -> np.ndarray:
    """Column positions of the k smallest keys of each row, in increasing key order."""
    n = keys.shape[1]
    part = np.argpartition(keys, k - 1, axis=1)[:, :k] if k < n else np.tile(np.arange(n), (keys.shape[0], 1))
    order = np.argsort(np.take_along_axis(keys, part, axis=1), axis=1, kind="stable")
    return np.take_along_axis(part, order, axis=1)


def _block_indices(rng, w: Workload, S: int, allow_future: bool) -> np.ndarray:
    """[S, Hkv, topk] int32 block indices for one sequence."""
    bs, topk, Hkv = w.block_size, w.topk, w.Hkv
    nblk = (S + bs - 1) // bs
    idx = np.full((S, Hkv, topk), -1, dtype=np.int32)
    for J in range(nblk):
        t0, t1 = J * bs, min(S, (J + 1) * bs)
        rows = (t1 - t0) * Hkv
        if w.select == "diag_uniform":
            # slot 0 = own (diagonal) block, then distinct uniform earlier blocks
            ncand = nblk if allow_future else J
            cand = np.array([c for c in range(ncand) if c != J], dtype=np.int64)
            k = min(topk - 1, len(cand))
            sel = np.full((rows, topk), -1, dtype=np.int64)
            sel[:, 0] = J
            if k > 0:
                keys = rng.random((rows, len(cand)))
                sel[:, 1:1 + k] = cand[_smallest_k(keys, k)]
        elif w.select == "zipf":
            # distinct blocks from [0, diag] (or all blocks), weight (b+1)^-s,
            # sequential weighted sampling without replacement via exponential keys
            ncand = nblk if allow_future else J + 1
            wts = (np.arange(ncand, dtype=np.float64) + 1.0) ** (-w.zipf_s)
            k = min(topk, ncand)
            u = rng.random((rows, ncand))
            keys = -np.log1p(-u) / wts
            sel = np.full((rows, topk), -1, dtype=np.int64)
            sel[:, :k] = _smallest_k(keys, k)
        else:
            raise ValueError(f"block selection {w.select!r}")
        idx[t0:t1] = sel.reshape(t1 - t0, Hkv, topk).astype(np.int32)
    if w.p_drop > 0:
        drop = rng.random(idx.shape) < w.p_drop
        idx[drop] = -1
    return idx


def _token_indices(rng, w: Workload, S: int) -> np.ndarray:
    """[S, Hkv, topk] int32 distinct token indices in [0, t] (uniform), -1 padded."""
    topk, Hkv = w.topk, w.Hkv
    idx = np.full((S, Hkv, topk), -1, dtype=np.int32)
    for t in range(S):
        n = t + 1
        for g in range(Hkv):
            keys = rng.random(n)
            if n <= topk:
                sel = np.argsort(keys, kind="stable")
            else:
                sel = np.argpartition(keys, topk - 1)[:topk]
            idx[t, g, :len(sel)] = sel
    return idx


def _cmp_indices(rng, w: Workload, S: int, any_pos: bool) -> np.ndarray:
    """[S, Hkv, cmp_topk] distinct compressed-row indices, -1 padded.

    By default each token draws from the compressed rows whose whole source
    group lies at or before it ((c+1)*ratio - 1 <= t); ``any_pos`` draws from
    every compressed row of the sequence instead (used by tests to exercise the
    compressed causal mask).
    """
    r, k, Hkv = w.cmp_ratio, w.cmp_topk, w.Hkv
    Tc = S // r
    idx = np.full((S, Hkv, k), -1, dtype=np.int32)
    for t in range(S):
        n = Tc if any_pos else (t + 1) // r
        if n == 0:
            continue
        for g in range(Hkv):
            keys = rng.random(n)
            if n <= k:
                sel = np.argsort(keys, kind="stable")
            else:
                sel = np.argpartition(keys, k - 1)[:k]
            idx[t, g, :len(sel)] = sel
    return idx


def make_inputs(w: Workload, *, allow_future: bool = False, cmp_any: bool = False,
                ori_len_range: tuple | None = None, dense: bool = True) -> dict:
    """Draw every input of workload ``w``.

    Returns a dict of numpy arrays.  bf16 tensors are uint16 bit patterns with
    shape [B, S, H, d] (BSND) or [T, H, d] (TND); index tensors are int32 with
    shape [..., Hkv, slots]; topk lengths are int32 [..., Hkv].

    Test-only knobs: ``allow_future`` lets block selections name blocks after
    the diagonal (the causal mask must then hide them); ``cmp_any`` draws cmp
    indices from all compressed rows; ``ori_len_range`` adds a per-row ori topk
    length drawn uniformly from the inclusive range.

    ``dense=False`` skips q, k / kv, v, dO and cmp_kv (the stream then serves
    the sinks and the index sets only): the benchmark draws those dense
    tensors on the GPU instead (``gen.torch_io.dense_on_device``), which the
    long-sequence workloads need to start within seconds.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed))
    lens = w.seq_lengths
    T = sum(lens)
    lead = (w.B, w.S) if w.layout == "BSND" else (T,)
    out: dict = {}

    if dense:
        out["q"] = _normal_bf16(rng, lead + (w.Hq, w.d_qk))
        if w.kv_shared:
            out["kv"] = _normal_bf16(rng, lead + (w.Hkv, w.d_qk))
        else:
            out["k"] = _normal_bf16(rng, lead + (w.Hkv, w.d_qk))
            out["v"] = _normal_bf16(rng, lead + (w.Hkv, w.d_v))
        out["do"] = _normal_bf16(rng, lead + (w.Hq, w.d_v), mul=w.do_scale)
    if w.sinks:
        out["sinks"] = rng.standard_normal(w.Hq, dtype=np.float32)

    starts = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)

    if w.topk > 0:
        parts = []
        for b, L in enumerate(lens):
            if w.mode == "block":
                parts.append(_block_indices(rng, w, L, allow_future))
            elif w.mode == "token":
                parts.append(_token_indices(rng, w, L))
            else:
                raise ValueError(f"ori indices in mode {w.mode!r}")
        idx = np.concatenate(parts, axis=0)
        out["ori_idx"] = idx.reshape(lead + (w.Hkv, w.topk))

    if w.cmp_topk > 0 or w.cmp_all:
        cmp_lens = [L // w.cmp_ratio for L in lens]
        if dense:
            kvkey = "kv" if w.kv_shared else "k"
            src = out[kvkey].reshape((T, w.Hkv, w.d_qk))
            cmp_parts = []
            for b, L in enumerate(lens):
                Tc = L // w.cmp_ratio
                seg = f32_from_bf16_bits(src[starts[b]:starts[b] + Tc * w.cmp_ratio]).astype(np.float64)
                pooled = seg.reshape(Tc, w.cmp_ratio, w.Hkv, w.d_qk).mean(axis=1)
                cmp_parts.append(bf16_bits_from_f32(pooled.astype(np.float32)))
            out["cmp_kv"] = np.concatenate(cmp_parts, axis=0)
        out["cu_seqlens_cmp"] = np.concatenate([[0], np.cumsum(cmp_lens)]).astype(np.int32)
        out["cmp_residual"] = np.array([L % w.cmp_ratio for L in lens], dtype=np.int32)
        if w.cmp_topk > 0:
            cidx = np.concatenate([_cmp_indices(rng, w, L, cmp_any) for L in lens], axis=0)
            out["cmp_idx"] = cidx.reshape(lead + (w.Hkv, w.cmp_topk))

    if ori_len_range is not None and w.topk > 0:
        lo, hi = ori_len_range
        out["ori_topk_len"] = rng.integers(lo, hi + 1, size=lead + (w.Hkv,)).astype(np.int32)

    if w.cmp_topk > 0:
        lo, hi = w.cmp_len_range
        raw = rng.integers(lo, hi + 1, size=(T, w.Hkv))
        cap = np.empty((T, w.Hkv), dtype=np.int64)
        for b, L in enumerate(lens):
            t = np.arange(L)
            n = (np.full(L, L // w.cmp_ratio) if cmp_any else (t + 1) // w.cmp_ratio)
            cap[starts[b]:starts[b] + L] = n[:, None]
        out["cmp_topk_len"] = np.minimum(raw, cap).astype(np.int32).reshape(lead + (w.Hkv,))

    if w.used:
        assert len(w.used) == len(lens)
        out["seqused_q"] = np.asarray(w.used, dtype=np.int32)
        out["seqused_kv"] = np.asarray(w.used, dtype=np.int32)
        if w.cmp_topk > 0 or w.cmp_all:
            out["seqused_cmp"] = np.asarray([u // w.cmp_ratio for u in w.used], dtype=np.int32)

    if w.layout == "TND":
        out["cu_seqlens_q"] = starts.astype(np.int32)
        out["cu_seqlens_kv"] = starts.astype(np.int32)
    return out


def make_paged_inputs(seed: int, *, B: int, s_q: int, kv_lens, page: int, Hq: int, Hkv: int, d_qk: int, d_v: int,
                      kv_shared: bool, block_size: int, topk: int, sinks: bool = True, spare_pages: int = 3) -> dict:
    """Decode-style inputs over a paged KV cache: s_q query tokens at the end of each
    of B sequences (lengths kv_lens), the cache's pages in shuffled order behind a
    per-sequence block table, and causal index sets (block_size-row blocks with the
    diagonal block first, or tokens) drawn over each query's visible prefix.  Dense
    tensors fp32 N(0, 1) -> bf16 (RNE) bit patterns; indices int32, -1 padded."""
    rng = np.random.default_rng(seed)
    kv_lens = np.asarray(kv_lens, dtype=np.int64)
    max_pages = int(-(-int(kv_lens.max()) // page))
    n_pages = B * max_pages + spare_pages
    table = rng.permutation(n_pages)[:B * max_pages].reshape(B, max_pages).astype(np.int32)
    rows = n_pages * page
    out = {"q": bf16_bits_from_f32(rng.standard_normal((B * s_q, Hq, d_qk), dtype=np.float32))}
    if kv_shared:
        out["kv"] = bf16_bits_from_f32(rng.standard_normal((rows, Hkv, d_qk), dtype=np.float32))
    else:
        out["k"] = bf16_bits_from_f32(rng.standard_normal((rows, Hkv, d_qk), dtype=np.float32))
        out["v"] = bf16_bits_from_f32(rng.standard_normal((rows, Hkv, d_v), dtype=np.float32))
    idx = np.full((B * s_q, Hkv, topk), -1, dtype=np.int32)
    for b in range(B):
        for t in range(s_q):
            ta = t + int(kv_lens[b]) - s_q                       # the query's position in its sequence
            for g in range(Hkv):
                if block_size > 1:
                    diag = ta // block_size
                    rest = rng.permutation(diag)[:topk - 1]
                    sel = np.concatenate([[diag], rest])
                else:
                    sel = rng.permutation(ta + 1)[:topk]
                idx[b * s_q + t, g, :len(sel)] = sel
    out["ori_idx"] = idx
    out["block_table"] = table
    out["seqused_kv"] = kv_lens.astype(np.int32)
    if sinks:
        out["sinks"] = rng.standard_normal(Hq).astype(np.float32)
    out["_meta"] = dict(B=B, s_q=s_q, s_kv=max_pages * page, t_kv=rows, page=page, Hq=Hq, Hkv=Hkv, d_qk=d_qk,
                        d_v=d_v, kv_shared=kv_shared, block_size=block_size, topk=topk)
    return out


def make_indexer_inputs(seed: int, *, lens, H: int, d: int, topk: int, layout: str = "TND") -> dict:
    """Inputs of the indexer KL-loss backward: q [T, H, d] and k [T, d] (fp32 N(0, 1) ->
    bf16 bits), w [T, H] fp32 N(0, 1) / sqrt(H), token indices drawn over each token's
    visible prefix [0, t] (-1 padded, in random slot order), a per-token usable length,
    and a target p: uniform random weights on the usable filled slots, normalised to 1."""
    rng = np.random.default_rng(seed)
    T = sum(lens)
    q = bf16_bits_from_f32(rng.standard_normal((T, H, d), dtype=np.float32))
    k = bf16_bits_from_f32(rng.standard_normal((T, d), dtype=np.float32))
    w = (rng.standard_normal((T, H)) / np.sqrt(H)).astype(np.float32)
    idx = np.full((T, topk), -1, dtype=np.int32)
    off = 0
    for L in lens:
        for t in range(L):
            sel = rng.permutation(t + 1)[:topk]
            row = np.full(topk, -1, dtype=np.int32)
            row[:len(sel)] = sel
            idx[off + t] = rng.permutation(row)
        off += L
    tlen = rng.integers(topk // 2, topk + 1, T).astype(np.int32)
    p = rng.random((T, topk)).astype(np.float32)
    usable = (idx >= 0) & (np.arange(topk)[None, :] < tlen[:, None])
    p = np.where(usable, p, 0.0).astype(np.float32)
    s = p.sum(axis=1, keepdims=True)
    p = np.where(s > 0, p / np.where(s > 0, s, 1), 0.0).astype(np.float32)
    starts = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return dict(q=q, k=k, w=w, idx=idx, topk_len=tlen, p=p, cu_seqlens=starts, lens=tuple(lens), layout=layout)
