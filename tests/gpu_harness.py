"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
on seeded inputs and compare with the float64 oracle.

Tolerances (fixed by the acceptance criteria of this build): bf16 and fp32
gradient tensors need max|err| <= 2e-2 * max|ref| and cosine >= 0.9999; lse
needs |err| <= 1e-4 absolute (and +inf exactly where the oracle has +inf);
visible index sets must match exactly.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from gen import f32_from_bf16_bits, make_inputs
from gen.torch_io import bf16_bits, to_torch
from top_sparse_attention_attn_b200 import SparseAttention

REL_TOL = 2e-2
COS_MIN = 0.9999
LSE_ATOL = 1e-4


def widen(bits) -> np.ndarray:
    return f32_from_bf16_bits(np.asarray(bits)).astype(np.float64)


def check_close(name: str, got, ref, rel=REL_TOL, cos_min=COS_MIN):
    """Element-wise comparison with the bf16 rule (inputs float64 arrays)."""
    got = np.asarray(got, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    assert got.shape == ref.shape, name
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    mref = np.abs(ref).max() if ref.size else 0.0
    err = np.abs(got - ref).max() if ref.size else 0.0
    assert err <= rel * mref + 1e-30, f"{name}: max|err| {err:.4g} > {rel} * max|ref| {mref:.4g}"
    ng, nr = np.linalg.norm(got), np.linalg.norm(ref)
    if nr == 0.0:
        assert ng == 0.0, f"{name}: reference is zero, got norm {ng}"
        return 1.0
    cos = float(got @ ref / (ng * nr)) if ng > 0 else 0.0
    assert cos >= cos_min, f"{name}: cosine {cos:.6f} < {cos_min}"
    return cos


def check_lse(name: str, got, ref):
    got = np.asarray(got, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    inf_r, inf_g = np.isinf(ref), np.isinf(got)
    assert np.array_equal(inf_r, inf_g), f"{name}: +inf rows differ ({inf_r.sum()} vs {inf_g.sum()})"
    assert np.all(got[inf_g] > 0)
    if (~inf_r).any():
        err = np.abs(got[~inf_r] - ref[~inf_r]).max()
        assert err <= LSE_ATOL, f"{name}: lse max|err| {err:.3g} > {LSE_ATOL}"


def device_problem(w, inputs, flags: int = 0):
    t = to_torch(inputs, "cuda")
    return SparseAttention.from_workload(w, t, flags=flags), t


def oracle_codes(p: oracle.Problem, tq: int, g: int) -> np.ndarray:
    ori, cmp = oracle.visible_rows(p, tq, g)
    return np.sort(np.concatenate([ori, np.asarray(cmp, dtype=np.int64) | 0x40000000]))


def max_visible_rows(w) -> int:
    n = 0
    if w.topk:
        n += w.topk * max(w.block_size, 1) if w.block_size > 1 else w.topk
    else:
        n += (w.win_left + w.win_right + 1) if w.ori_mask == "band" else max(w.seq_lengths)
    n += w.cmp_topk if w.cmp_topk else (max(w.seq_lengths) // w.cmp_ratio if w.cmp_all else 0)
    return n


def check_resolve(sa: SparseAttention, p: oracle.Problem, w, units):
    max_rows = max_visible_rows(w)
    rows, counts = sa.debug_resolve(max_rows)
    rows, counts = rows.cpu().numpy(), counts.cpu().numpy()
    for tq, g in units:
        u = tq * w.Hkv + g
        ref = oracle_codes(p, tq, g)
        assert counts[u] == len(ref), f"unit {(tq, g)}: {counts[u]} visible rows, oracle {len(ref)}"
        got = np.sort(rows[u, :counts[u]].astype(np.int64))
        assert np.array_equal(got, ref), f"unit {(tq, g)}: visible rows differ"


def grads_to_host(grads: dict) -> dict:
    out = {}
    for k, v in grads.items():
        out[k] = v.float().cpu().numpy() if k == "dsinks" else bf16_bits(v)
    return out


def compare_grads(tag: str, got: dict, ref: dict, T: int, w):
    for key in ref:
        if key == "dq":
            continue
        g = got[key]
        r = ref[key]
        if key == "dsinks":
            check_close(f"{tag}:{key}", g, r)
        else:
            check_close(f"{tag}:{key}", widen(g), widen(r))
    check_close(f"{tag}:dq", widen(got["dq"]).reshape(T, -1), widen(ref["dq"]).reshape(T, -1))


def run_full_comparison(w, gen_kwargs=None, flags=0, inputs=None):
    """Small workload: every output element compared with the oracle (on ``inputs``
    when given, else on the workload's generated inputs)."""
    if inputs is None:
        inputs = make_inputs(w, **(gen_kwargs or {}))
    p = oracle.Problem.from_inputs(w, inputs)
    T = w.T
    sa, t = device_problem(w, inputs, flags)

    # forward
    O_ref, lse_ref = oracle.forward(p)
    o, lse = sa.forward()
    torch.cuda.synchronize()
    check_close(f"{w.name}:O", widen(bf16_bits(o)).reshape(T, -1), widen(O_ref).reshape(T, -1))
    check_lse(f"{w.name}:lse", lse.cpu().numpy().reshape(T, -1), lse_ref)

    # resolved visible sets, bit-exact
    check_resolve(sa, p, w, p.all_units())

    # backward on the oracle's O and lse (as the workload prescribes)
    do = inputs["do"].reshape(T, w.Hq, w.d_v)
    ref = oracle.backward(p, O_ref, lse_ref, do)
    o_in = to_torch({"o": O_ref.reshape(o.shape)}, "cuda")["o"]
    lse_in = torch.from_numpy(np.ascontiguousarray(lse_ref.reshape(lse.shape))).cuda()
    grads = sa.backward(o_in, lse_in, t["do"])
    torch.cuda.synchronize()
    compare_grads(f"{w.name}:bwd", grads_to_host(grads), ref, T, w)

    # rowsum(dO o O) against the oracle's Delta
    delta = sa.delta(o_in, t["do"]).cpu().numpy().reshape(T, -1)
    ref_delta = (widen(O_ref).reshape(T, w.Hq, w.d_v) * widen(do)).sum(-1)
    np.testing.assert_allclose(delta, ref_delta, rtol=1e-5, atol=1e-5 * max(1.0, np.abs(ref_delta).max()))

    # end to end: GPU forward -> GPU backward
    grads2 = sa.backward(o, lse, t["do"])
    torch.cuda.synchronize()
    compare_grads(f"{w.name}:e2e", grads_to_host(grads2), ref, T, w)
    return p, sa


class UnitRows:
    """Array-like over sampled query tokens: rows[tq] is an [H, d] (or [H]) array."""

    def __init__(self):
        self.rows = {}

    def __getitem__(self, key):
        tq, hs = key
        return self.rows[tq][hs]


def contributor_units(w, inputs, b: int, g: int, ori_rows=None, cmp_rows=None):
    """Units of batch b / kv-head g whose selection may reach the given local rows (a superset)."""
    lens = w.seq_lengths
    start = int(np.sum(lens[:b]))
    L = lens[b]
    T = w.T
    toks = set()
    if ori_rows is not None and len(ori_rows):
        rmin = int(np.min(ori_rows))
        if w.topk:
            idx = inputs["ori_idx"].reshape(T, w.Hkv, -1)[start:start + L, g]
            targets = np.unique(np.asarray(ori_rows) // w.block_size)
            hit = np.isin(idx, targets).any(axis=1)
            toks.update((start + np.nonzero(hit)[0]).tolist())
        else:  # window: tokens whose band reaches the rows
            lo = max(0, rmin - w.win_right)
            hi = min(L - 1, int(np.max(ori_rows)) + w.win_left)
            toks.update(range(start + lo, start + hi + 1))
    if cmp_rows is not None and len(cmp_rows):
        cidx = inputs["cmp_idx"].reshape(T, w.Hkv, -1)[start:start + L, g]
        hit = np.isin(cidx, np.asarray(cmp_rows)).any(axis=1)
        toks.update((start + np.nonzero(hit)[0]).tolist())
    return [(tq, g) for tq in sorted(toks)]


def run_sampled(w, n_units=24, seed=0, tail_rows=64, inputs=None):
    """Full-size workload in the benchmark's launch configuration: GPU forward then
    backward on its own O / lse; sampled units and tail KV rows checked against the
    oracle run end to end on the same units."""
    if inputs is None:
        inputs = make_inputs(w)
    p = oracle.Problem.from_inputs(w, inputs)
    T, G = w.T, w.G
    sa, t = device_problem(w, inputs)
    o, lse = sa.forward()
    grads = sa.backward(o, lse, t["do"])
    torch.cuda.synchronize()

    rng = np.random.default_rng(seed)
    units = {(0, 0), (T - 1, w.Hkv - 1)}
    while len(units) < n_units:
        units.add((int(rng.integers(T)), int(rng.integers(w.Hkv))))
    units = sorted(units)

    # forward rows and dQ rows of the sampled units
    fw = oracle.forward(p, units=units)
    O_rows, L_rows = UnitRows(), UnitRows()
    for (tq, g), (ob, lb) in fw.items():
        O_rows.rows.setdefault(tq, np.zeros((w.Hq, w.d_v), dtype=np.uint16))[g * G:(g + 1) * G] = ob
        L_rows.rows.setdefault(tq, np.zeros(w.Hq, dtype=np.float32))[g * G:(g + 1) * G] = lb
    do = inputs["do"].reshape(T, w.Hq, w.d_v)
    bw = oracle.backward(p, O_rows, L_rows, do, units=units)
    o_h = o.view(T, w.Hq, w.d_v)
    lse_h = lse.view(T, w.Hq)
    dq_h = grads["dq"].view(T, w.Hq, w.d_qk)
    got_o, ref_o, got_l, ref_l, got_q, ref_q = [], [], [], [], [], []
    for (tq, g) in units:
        hs = slice(g * G, (g + 1) * G)
        got_o.append(widen(bf16_bits(o_h[tq, hs])))
        ref_o.append(widen(fw[(tq, g)][0]))
        got_l.append(lse_h[tq, hs].cpu().numpy())
        ref_l.append(fw[(tq, g)][1])
        got_q.append(widen(bf16_bits(dq_h[tq, hs])))
        ref_q.append(widen(bw["dq"][(tq, g)]))
    check_close(f"{w.name}:O[sampled]", np.concatenate(got_o), np.concatenate(ref_o))
    check_lse(f"{w.name}:lse[sampled]", np.concatenate(got_l), np.concatenate(ref_l))
    check_close(f"{w.name}:dQ[sampled]", np.concatenate(got_q), np.concatenate(ref_q))

    # tail KV rows of the last sequence, every kv-head: exact with all contributors
    b = w.n_batches - 1
    L = w.seq_lengths[b]
    start = int(np.sum(w.seq_lengths[:b]))
    rows = np.arange(max(0, L - tail_rows), L)
    crow = None
    if w.cmp_topk:
        Lc = L // w.cmp_ratio
        crow = np.arange(max(0, Lc - tail_rows // w.cmp_ratio), Lc)
    host = grads_to_host(grads)
    for g in range(w.Hkv):
        cu = contributor_units(w, inputs, b, g, ori_rows=rows, cmp_rows=crow)
        fw2 = oracle.forward(p, units=cu)
        O2, L2 = UnitRows(), UnitRows()
        for (tq, gg), (ob, lb) in fw2.items():
            O2.rows.setdefault(tq, np.zeros((w.Hq, w.d_v), dtype=np.uint16))[gg * G:(gg + 1) * G] = ob
            L2.rows.setdefault(tq, np.zeros(w.Hq, dtype=np.float32))[gg * G:(gg + 1) * G] = lb
        bw2 = oracle.backward(p, O2, L2, do, units=cu)
        for key in ("dk", "dv", "dkv"):
            if key in bw2:
                got = host[key].reshape(p.Tk, w.Hkv, -1)[start + rows, g]
                check_close(f"{w.name}:{key}[tail, g={g}]", widen(got), widen(bw2[key][start + rows, g]))
        if crow is not None:
            cstart = int(np.sum([x // w.cmp_ratio for x in w.seq_lengths[:b]]))
            got = host["dcmp"].reshape(p.Tc, w.Hkv, -1)[cstart + crow, g]
            check_close(f"{w.name}:dcmp[tail, g={g}]", widen(got), widen(bw2["dcmp"][cstart + crow, g]))
    return sa, o, lse, grads
