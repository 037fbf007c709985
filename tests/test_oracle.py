"""Pins for the float64 oracle, all on the CPU.

Each test checks the oracle against something other than its own formulas:
central finite differences of sum(O*dO), torch float64 autograd of an
independently written masked-dense forward, torch's scaled_dot_product_attention
on the dense special case, hand-worked closed forms (tests/golden), invariants
of softmax and of its gradient, and scalar brute force on tiny inputs.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import Problem

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# ----------------------------------------------------------------------------
# tiny problems in float64 (not bf16) with every selection feature switched on
# ----------------------------------------------------------------------------


def _tiny_params(mode: str, seed: int, dup: bool = False):
    rng = np.random.default_rng(seed)
    if mode == "block":
        lens, Hq, Hkv, dqk, dv, bs, topk = (13, 9), 4, 2, 6, 5, 4, 4
        T = sum(lens)
        par = dict(q=rng.standard_normal((T, Hq, dqk)), k=rng.standard_normal((T, Hkv, dqk)),
                   v=rng.standard_normal((T, Hkv, dv)))
        idx = np.full((T, Hkv, topk), -1, dtype=np.int64)
        off = 0
        for L in lens:
            nblk = (L + bs - 1) // bs
            for t in range(L):
                for g in range(Hkv):
                    sel = rng.permutation(nblk)[:rng.integers(1, topk + 1)]   # future blocks too
                    idx[off + t, g, :len(sel)] = sel
                    if len(sel) < topk and rng.random() < 0.5:
                        idx[off + t, g] = rng.permutation(idx[off + t, g])      # -1 in the middle
            off += L
        if dup:
            idx[5, 0, :2] = [0, 0]
        meta = dict(lens=lens, Hq=Hq, Hkv=Hkv, dqk=dqk, dv=dv, bs=bs, shared=False,
                    ori_idx=idx, ori_len=rng.integers(0, topk + 1, (T, Hkv)),
                    ori_mask="causal", scale=0.7)
    elif mode == "token":
        lens, Hq, Hkv, dqk, dv, topk = (11, 7), 4, 1, 6, 4, 5
        T = sum(lens)
        par = dict(q=rng.standard_normal((T, Hq, dqk)), kv=rng.standard_normal((T, Hkv, dqk)))
        idx = np.full((T, Hkv, topk), -1, dtype=np.int64)
        off = 0
        for L in lens:
            for t in range(L):
                sel = rng.permutation(L)[:rng.integers(0, topk + 1)]          # future tokens too
                idx[off + t, 0, :len(sel)] = sel
            off += L
        if dup:
            idx[4, 0, :3] = [1, 1, 0]
        meta = dict(lens=lens, Hq=Hq, Hkv=Hkv, dqk=dqk, dv=dv, bs=1, shared=True,
                    ori_idx=idx, ori_len=None, ori_mask="causal", scale=0.45)
    elif mode == "swa_cmp":
        lens, Hq, Hkv, dqk, dv, ratio, ctopk = (14, 10), 4, 1, 6, 4, 4, 3
        T = sum(lens)
        clens = tuple(L // ratio for L in lens)
        Tc = sum(clens)
        par = dict(q=rng.standard_normal((T, Hq, dqk)), kv=rng.standard_normal((T, Hkv, dqk)),
                   cmp_kv=rng.standard_normal((Tc, Hkv, dqk)), sinks=rng.standard_normal(Hq))
        cidx = np.full((T, Hkv, ctopk), -1, dtype=np.int64)
        off = 0
        for L, C in zip(lens, clens):
            for t in range(L):
                sel = rng.permutation(C)[:rng.integers(0, ctopk + 1)]         # causally invalid too
                cidx[off + t, 0, :len(sel)] = sel
            off += L
        meta = dict(lens=lens, Hq=Hq, Hkv=Hkv, dqk=dqk, dv=dv, bs=1, shared=True, ori_idx=None,
                    ori_len=None, ori_mask="band", win_left=3, win_right=1, cmp_lens=clens,
                    cmp_idx=cidx, cmp_len=rng.integers(0, ctopk + 1, (T, Hkv)), ratio=ratio,
                    scale=0.5)
    elif mode == "cfa":
        # SparseFlashMlaGrad Stage 1, "else" (CFA): the window over the original KV
        # concatenated with every compressed row (no cmp indices)
        lens, Hq, Hkv, dqk, dv, ratio = (14, 10), 4, 1, 6, 4, 3
        T = sum(lens)
        clens = tuple(L // ratio for L in lens)
        par = dict(q=rng.standard_normal((T, Hq, dqk)), kv=rng.standard_normal((T, Hkv, dqk)),
                   cmp_kv=rng.standard_normal((sum(clens), Hkv, dqk)), sinks=rng.standard_normal(Hq))
        meta = dict(lens=lens, Hq=Hq, Hkv=Hkv, dqk=dqk, dv=dv, bs=1, shared=True, ori_idx=None,
                    ori_len=None, ori_mask="band", win_left=2, win_right=0, cmp_lens=clens, ratio=ratio,
                    cfa=True, scale=0.5)
    else:
        raise ValueError(mode)
    par["do"] = rng.standard_normal((sum(meta["lens"]), meta["Hq"], meta["dv"]))
    return par, meta


def _build(par, meta) -> Problem:
    dv = meta["dv"]
    if meta["shared"]:
        k_ori, v_ori = par["kv"], par["kv"][..., :dv]
    else:
        k_ori, v_ori = par["k"], par["v"]
    kw = {}
    if "cmp_kv" in par:
        kw = dict(k_cmp=par["cmp_kv"], v_cmp=par["cmp_kv"][..., :dv], cmp_lens=meta["cmp_lens"],
                  cmp_ratio=meta["ratio"])
        if "cmp_idx" in meta:
            kw.update(cmp_idx=meta["cmp_idx"], cmp_topk_len=meta["cmp_len"])
    return Problem(q=par["q"], k_ori=k_ori, v_ori=v_ori, kv_shared=meta["shared"],
                   q_lens=meta["lens"], kv_lens=meta["lens"], Hq=meta["Hq"], Hkv=meta["Hkv"],
                   d_qk=meta["dqk"], d_v=dv, scale=meta["scale"], block_size=meta["bs"],
                   ori_idx=meta["ori_idx"], ori_topk_len=meta["ori_len"],
                   ori_mask=meta["ori_mask"], win_left=meta.get("win_left", 0),
                   win_right=meta.get("win_right", 0), sinks=par.get("sinks"), **kw)


def _loss(par, meta) -> float:
    p = _build(par, meta)
    O, _ = oracle.forward(p, rounded=False)
    return float((O * par["do"]).sum())


def _grads(par, meta) -> dict:
    p = _build(par, meta)
    O, lse = oracle.forward(p, rounded=False)
    r = oracle.backward(p, O, lse, par["do"], rounded=False)
    out = {"q": r["dq"]}
    if meta["shared"]:
        out["kv"] = r["dkv"]
    else:
        out["k"], out["v"] = r["dk"], r["dv"]
    if "dcmp" in r:
        out["cmp_kv"] = r["dcmp"]
    if "dsinks" in r:
        out["sinks"] = r["dsinks"]
    return out


MODES = ["block", "token", "swa_cmp", "cfa"]


# ----------------------------------------------------------------------------
# 1. central finite differences of L = sum(O * dO)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("mode", MODES)
def test_backward_matches_finite_differences(mode):
    par, meta = _tiny_params(mode, seed=11)
    an = _grads(par, meta)
    h = 1e-6
    for name, g in an.items():
        x = par[name]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = x[i]
            x[i] = old + h
            lp = _loss(par, meta)
            x[i] = old - h
            lm = _loss(par, meta)
            x[i] = old
            fd[i] = (lp - lm) / (2 * h)
        scale = max(1.0, np.abs(g).max())
        err = np.abs(fd - g).max() / scale
        assert err < 1e-6, f"{mode}: d{name} differs from finite differences by {err:.3g}"
        assert np.abs(g).max() > 0, f"{mode}: d{name} is identically zero"


def test_backward_with_duplicate_indices_matches_finite_differences():
    for mode in ("block", "token"):
        par, meta = _tiny_params(mode, seed=5, dup=True)
        an = _grads(par, meta)
        h = 1e-6
        key = "k" if mode == "block" else "kv"
        x = par[key]
        for i in [(0, 0, 0), (1, 0, 2), (0, 0, 3)]:
            old = x[i]
            x[i] = old + h
            lp = _loss(par, meta)
            x[i] = old - h
            lm = _loss(par, meta)
            x[i] = old
            assert abs((lp - lm) / (2 * h) - an[key][i]) < 1e-6


# ----------------------------------------------------------------------------
# 2. torch float64 autograd of an independently written masked-dense forward
# ----------------------------------------------------------------------------

def _selection_counts(meta, tq, g, b, t, L, off):
    """How many times each key row of the sequence is selected, from the definition."""
    counts = np.zeros(L)
    if meta["ori_idx"] is not None:
        nslot = meta["ori_idx"].shape[2]
        if meta["ori_len"] is not None:
            nslot = min(nslot, meta["ori_len"][tq, g])
        for i in range(nslot):
            x = meta["ori_idx"][tq, g, i]
            if x < 0:
                continue
            for r in range(x * meta["bs"], x * meta["bs"] + meta["bs"]):
                if r < L:
                    counts[r] += 1
    else:
        counts[:] = 1
    for r in range(L):
        if meta["ori_mask"] == "causal" and r > t:
            counts[r] = 0
        if meta["ori_mask"] == "band" and not (t - meta["win_left"] <= r <= t + meta["win_right"]):
            counts[r] = 0
    ccounts = None
    if "cmp_idx" in meta:
        C = meta["cmp_lens"][b]
        ccounts = np.zeros(C)
        for i in range(min(meta["cmp_idx"].shape[2], meta["cmp_len"][tq, g])):
            c = meta["cmp_idx"][tq, g, i]
            if c >= 0 and (c + 1) * meta["ratio"] - 1 <= t:
                ccounts[c] += 1
    elif meta.get("cfa"):
        C = meta["cmp_lens"][b]
        ccounts = np.array([1.0 if (c + 1) * meta["ratio"] - 1 <= t else 0.0 for c in range(C)])
    return counts, ccounts


def _torch_forward(tp, meta):
    """Masked-dense attention with multiplicity weights, per sequence, in torch float64."""
    dv, G = meta["dv"], meta["Hq"] // meta["Hkv"]
    O = torch.zeros(tp["q"].shape[0], meta["Hq"], dv, dtype=torch.float64)
    outs = []
    off, coff = 0, 0
    for b, L in enumerate(meta["lens"]):
        for t in range(L):
            tq = off + t
            for g in range(meta["Hkv"]):
                hs = slice(g * G, (g + 1) * G)
                if meta["shared"]:
                    K = tp["kv"][off:off + L, g]
                    V = K[:, :dv]
                else:
                    K, V = tp["k"][off:off + L, g], tp["v"][off:off + L, g]
                counts, ccounts = _selection_counts(meta, tq, g, b, t, L, off)
                logw = torch.log(torch.tensor(counts))               # -inf where unselected
                s = meta["scale"] * tp["q"][tq, hs] @ K.T + logw
                vals = [V]
                cols = [s]
                if ccounts is not None:
                    C = meta["cmp_lens"][b]
                    Kc = tp["cmp_kv"][coff:coff + C, g]
                    cols.append(meta["scale"] * tp["q"][tq, hs] @ Kc.T + torch.log(torch.tensor(ccounts)))
                    vals.append(Kc[:, :dv])
                if "sinks" in tp:
                    cols.append(tp["sinks"][hs][:, None])
                    vals.append(torch.zeros(1, dv, dtype=torch.float64))
                s_all = torch.cat(cols, dim=1)
                v_all = torch.cat(vals, dim=0)
                if torch.isinf(s_all).all():
                    outs.append((tq, hs, torch.zeros(G, dv, dtype=torch.float64)))
                    continue
                outs.append((tq, hs, torch.softmax(s_all, dim=1) @ v_all))
        off += L
        if "cmp_lens" in meta:
            coff += meta["cmp_lens"][b]
    for tq, hs, o in outs:
        O[tq, hs] = o
    return O


@pytest.mark.parametrize("mode", MODES)
def test_forward_and_backward_match_torch_autograd(mode):
    par, meta = _tiny_params(mode, seed=23)
    tp = {k: torch.tensor(v, requires_grad=(k != "do")) for k, v in par.items()}
    O_t = _torch_forward(tp, meta)
    (O_t * tp["do"]).sum().backward()

    p = _build(par, meta)
    O, lse = oracle.forward(p, rounded=False)
    np.testing.assert_allclose(O, O_t.detach().numpy(), rtol=0, atol=1e-12)
    r = oracle.backward(p, O, lse, par["do"], rounded=False)
    pairs = [("dq", "q")]
    pairs += [("dkv", "kv")] if meta["shared"] else [("dk", "k"), ("dv", "v")]
    if "cmp_kv" in par:
        pairs.append(("dcmp", "cmp_kv"))
    if "sinks" in par:
        pairs.append(("dsinks", "sinks"))
    for ours, theirs in pairs:
        ref = tp[theirs].grad.numpy()
        np.testing.assert_allclose(r[ours], ref, rtol=0, atol=1e-10 * max(1, np.abs(ref).max()),
                                   err_msg=f"{mode}: {ours}")


# ----------------------------------------------------------------------------
# 3. dense special case == torch scaled_dot_product_attention
# ----------------------------------------------------------------------------

def _sdpa_case(kind, seed=3):
    rng = np.random.default_rng(seed)
    L, Hq, Hkv, dqk, dv, bs = 24, 4, 2, 8, 8, 4
    G = Hq // Hkv
    q = rng.standard_normal((L, Hq, dqk))
    if kind == "block_all":
        k, v = rng.standard_normal((L, Hkv, dqk)), rng.standard_normal((L, Hkv, dv))
        nblk = L // bs
        idx = np.stack([np.stack([rng.permutation(nblk) for _ in range(Hkv)]) for _ in range(L)])
        p = Problem(q=q, k_ori=k, v_ori=v, kv_shared=False, q_lens=[L], kv_lens=[L], Hq=Hq,
                    Hkv=Hkv, d_qk=dqk, d_v=dv, scale=0.3, block_size=bs, ori_idx=idx)
        mask = torch.ones(L, L, dtype=torch.bool).tril()
    elif kind == "token_all":
        kv = rng.standard_normal((L, Hkv, dqk))
        k, v = kv, kv[..., :dv]
        idx = np.stack([np.stack([rng.permutation(L) for _ in range(Hkv)]) for _ in range(L)])
        p = Problem(q=q, k_ori=k, v_ori=v, kv_shared=True, q_lens=[L], kv_lens=[L], Hq=Hq,
                    Hkv=Hkv, d_qk=dqk, d_v=dv, scale=0.3, block_size=1, ori_idx=idx)
        mask = torch.ones(L, L, dtype=torch.bool).tril()
    elif kind == "swa":
        kv = rng.standard_normal((L, Hkv, dqk))
        k, v = kv, kv[..., :dv]
        p = Problem(q=q, k_ori=k, v_ori=v, kv_shared=True, q_lens=[L], kv_lens=[L], Hq=Hq,
                    Hkv=Hkv, d_qk=dqk, d_v=dv, scale=0.3, ori_mask="band", win_left=5, win_right=2)
        mask = torch.ones(L, L, dtype=torch.bool).tril(2).triu(-5)
    else:
        raise ValueError(kind)
    return p, q, k, v, mask, G


@pytest.mark.parametrize("kind", ["block_all", "token_all", "swa"])
def test_dense_special_case_equals_sdpa(kind):
    p, q, k, v, mask, G = _sdpa_case(kind)
    rng = np.random.default_rng(9)
    dO = rng.standard_normal((p.T, p.Hq, p.d_v))
    tq = torch.tensor(q.transpose(1, 0, 2), requires_grad=True)                 # [H, L, d]
    tk = torch.tensor(np.ascontiguousarray(k.transpose(1, 0, 2)), requires_grad=True)
    tv = torch.tensor(np.ascontiguousarray(v.transpose(1, 0, 2)), requires_grad=True)
    o = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(G, 0), tv.repeat_interleave(G, 0), attn_mask=mask, scale=0.3)
    (o * torch.tensor(dO.transpose(1, 0, 2))).sum().backward()

    O, lse = oracle.forward(p, rounded=False)
    np.testing.assert_allclose(O, o.detach().numpy().transpose(1, 0, 2), rtol=0, atol=1e-12)
    r = oracle.backward(p, O, lse, dO, rounded=False)
    np.testing.assert_allclose(r["dq"], tq.grad.numpy().transpose(1, 0, 2), atol=1e-11)
    if p.kv_shared:
        ref = tk.grad.numpy().transpose(1, 0, 2).copy()
        ref[..., :p.d_v] += tv.grad.numpy().transpose(1, 0, 2)
        np.testing.assert_allclose(r["dkv"], ref, atol=1e-11)
    else:
        np.testing.assert_allclose(r["dk"], tk.grad.numpy().transpose(1, 0, 2), atol=1e-11)
        np.testing.assert_allclose(r["dv"], tv.grad.numpy().transpose(1, 0, 2), atol=1e-11)


# ----------------------------------------------------------------------------
# 4. hand-worked closed forms (tests/golden/worked_examples.json)
# ----------------------------------------------------------------------------

def _num(x):
    if isinstance(x, str):
        env = {"ln3": math.log(3.0), "ln4": math.log(4.0), "ln5": math.log(5.0)}
        return float(eval(x, {"__builtins__": {}}, env))
    return float(x)


def test_worked_examples():
    with open(os.path.join(GOLDEN, "worked_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q = np.array([[[_num(x) for x in c["q"]]]])                                  # [1, 1, 1]
        k = np.array([[[_num(x) for x in row]] for row in c["k"]])                  # [2, 1, 1]
        v = np.array([[[_num(x) for x in row]] for row in c["v"]])                  # [2, 1, 2]
        # the query sits at position 1 of a 2-token sequence; token 0's row is empty of interest
        qq = np.concatenate([np.zeros_like(q), q])
        idx = np.array([[[-1, -1]], [[0, 1]]])
        sinks = None if c["sink"] is None else np.array([c["sink"]])
        p = Problem(q=qq, k_ori=k, v_ori=v, kv_shared=False, q_lens=[2], kv_lens=[2], Hq=1,
                    Hkv=1, d_qk=1, d_v=2, scale=1.0, block_size=1, ori_idx=idx, sinks=sinks)
        O, lse = oracle.forward(p, rounded=False)
        e = c["expect"]
        assert abs(lse[1, 0] - _num(e["lse"])) < 1e-15
        np.testing.assert_allclose(O[1, 0], e["o"], atol=1e-15)
        dO = np.zeros((2, 1, 2))
        dO[1, 0] = c["do"]
        r = oracle.backward(p, O, lse, dO, units=[(1, 0)], rounded=False)
        np.testing.assert_allclose(r["dq"][(1, 0)][0], [_num(x) for x in e["dq"]], atol=1e-15)
        np.testing.assert_allclose(r["dk"][:, 0], e["dk"], atol=1e-15)
        np.testing.assert_allclose(r["dv"][:, 0], e["dv"], atol=1e-15)
        if e["dsink"] is not None:
            assert abs(r["dsinks"][0] - e["dsink"]) < 1e-15


def test_closed_form_single_key():
    """One visible key, no sink: P = 1, O = v, dS = 0 so dQ = dK = 0 and dV = sum of dO."""
    rng = np.random.default_rng(1)
    L, H, d = 9, 3, 5
    kv = rng.standard_normal((L, 1, d))
    idx = np.zeros((L, 1, 1), dtype=np.int64)                                        # all pick row 0
    p = Problem(q=rng.standard_normal((L, H, d)), k_ori=kv, v_ori=kv, kv_shared=True,
                q_lens=[L], kv_lens=[L], Hq=H, Hkv=1, d_qk=d, d_v=d, scale=0.8, ori_idx=idx)
    O, lse = oracle.forward(p, rounded=False)
    np.testing.assert_allclose(O, np.broadcast_to(kv[0, 0], O.shape), atol=1e-15)
    np.testing.assert_allclose(lse, 0.8 * np.einsum("thd,d->th", p.q, kv[0, 0]), atol=1e-14)
    dO = rng.standard_normal((L, H, d))
    r = oracle.backward(p, O, lse, dO, rounded=False)
    assert np.abs(r["dq"]).max() < 1e-14
    expect = np.zeros((L, 1, d))
    expect[0, 0] = dO.sum(axis=(0, 1))                                               # dV part; dK part 0
    np.testing.assert_allclose(r["dkv"], expect, atol=1e-13)


def test_closed_form_zero_query_is_uniform():
    rng = np.random.default_rng(2)
    L, H, d = 10, 2, 4
    k, v = rng.standard_normal((L, 1, d)), rng.standard_normal((L, 1, d))
    p = Problem(q=np.zeros((L, H, d)), k_ori=k, v_ori=v, kv_shared=False, q_lens=[L], kv_lens=[L],
                Hq=H, Hkv=1, d_qk=d, d_v=d, scale=1.0, block_size=1,
                ori_idx=np.tile(np.arange(L)[None, None, :], (L, 1, 1)))
    O, lse = oracle.forward(p, rounded=False)
    for t in range(L):
        np.testing.assert_allclose(lse[t], math.log(t + 1), atol=1e-14)
        np.testing.assert_allclose(O[t, 0], v[:t + 1, 0].mean(axis=0), atol=1e-14)


def test_empty_rows():
    """No visible key: without sink lse = +inf, O = 0, zero grads; with sink lse = sink."""
    rng = np.random.default_rng(4)
    L, H, d = 6, 2, 3
    k, v = rng.standard_normal((L, 1, d)), rng.standard_normal((L, 1, d))
    idx = np.full((L, 1, 2), -1)
    for sinks in (None, np.array([0.3, -1.2])):
        p = Problem(q=rng.standard_normal((L, H, d)), k_ori=k, v_ori=v, kv_shared=False,
                    q_lens=[L], kv_lens=[L], Hq=H, Hkv=1, d_qk=d, d_v=d, scale=1.0, ori_idx=idx,
                    sinks=sinks)
        O, lse = oracle.forward(p, rounded=False)
        assert np.all(O == 0)
        if sinks is None:
            assert np.all(np.isinf(lse)) and np.all(lse > 0)
        else:
            np.testing.assert_allclose(lse, np.broadcast_to(sinks, lse.shape))
        r = oracle.backward(p, O, lse, rng.standard_normal((L, H, d)), rounded=False)
        assert np.all(r["dq"] == 0) and np.all(r["dk"] == 0) and np.all(r["dv"] == 0)
        if sinks is not None:
            assert np.all(r["dsinks"] == 0)


# ----------------------------------------------------------------------------
# 5. invariants
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("mode", MODES)
def test_softmax_rows_and_dS_rowsums(mode):
    par, meta = _tiny_params(mode, seed=31)
    p = _build(par, meta)
    O, lse = oracle.forward(p, rounded=False)
    checked = 0
    for tq in range(p.T):
        for g in range(p.Hkv):
            hs = slice(g * p.G, (g + 1) * p.G)
            if np.isinf(lse[tq, hs]).any():
                continue
            r = oracle.unit_backward(p, tq, g, O[tq, hs], lse[tq, hs], par["do"][tq, hs])
            total = r["P"].sum(axis=1) + (r["P_sink"] if "P_sink" in r else 0.0)
            np.testing.assert_allclose(total, 1.0, atol=1e-13)
            rows = r["dS"].sum(axis=1) + (r["dSinks"] if "dSinks" in r else 0.0)
            np.testing.assert_allclose(rows, 0.0, atol=1e-12)
            checked += 1
    assert checked > 10


def test_masked_and_invalid_rows_contribute_nothing():
    par, meta = _tiny_params("block", seed=41)
    p = _build(par, meta)
    O, lse = oracle.forward(p, rounded=False)
    r = oracle.backward(p, O, lse, par["do"], rounded=False)
    # rows no unit can see: perturbing them changes nothing and their gradients are exactly 0
    seen = np.zeros((p.T, p.Hkv), dtype=bool)
    for tq in range(p.T):
        for g in range(p.Hkv):
            ori, _ = oracle.visible_rows(p, tq, g)
            seen[p.kv_start[p.batch_of(tq)] + ori, g] = True
    unseen = ~seen
    assert unseen.any()
    assert np.all(r["dk"][unseen] == 0) and np.all(r["dv"][unseen] == 0)
    par2 = {k: v.copy() for k, v in par.items()}
    par2["k"][unseen] += 100.0
    par2["v"][unseen] -= 50.0
    O2, lse2 = oracle.forward(_build(par2, meta), rounded=False)
    assert np.array_equal(O, O2) and np.array_equal(lse, lse2)


@pytest.mark.parametrize("mode", ["block", "token"])
def test_slot_order_does_not_matter(mode):
    par, meta = _tiny_params(mode, seed=51)
    g1 = _grads(par, meta)
    rng = np.random.default_rng(0)
    meta2 = dict(meta)
    idx = meta["ori_idx"].copy()
    if meta["ori_len"] is not None:
        # permute only inside the usable prefix so the selected set is unchanged
        for tq in range(idx.shape[0]):
            for g in range(idx.shape[1]):
                n = meta["ori_len"][tq, g]
                idx[tq, g, :n] = rng.permutation(idx[tq, g, :n])
    else:
        idx = np.stack([[rng.permutation(row) for row in tok] for tok in idx])
    meta2["ori_idx"] = idx
    g2 = _grads(par, meta2)
    for k in g1:
        np.testing.assert_allclose(g1[k], g2[k], atol=1e-12)


def test_gqa_kv_grad_is_sum_over_heads():
    par, meta = _tiny_params("block", seed=61)
    full = _grads(par, meta)
    G = meta["Hq"] // meta["Hkv"]
    dk = np.zeros_like(full["k"])
    dv = np.zeros_like(full["v"])
    for g in range(meta["Hkv"]):
        for j in range(G):
            h = g * G + j
            m1 = dict(meta, Hq=1, Hkv=1, ori_idx=meta["ori_idx"][:, g:g + 1],
                      ori_len=meta["ori_len"][:, g:g + 1])
            p1 = dict(q=par["q"][:, h:h + 1], k=par["k"][:, g:g + 1], v=par["v"][:, g:g + 1],
                      do=par["do"][:, h:h + 1])
            r1 = _grads(p1, m1)
            dk[:, g] += r1["k"][:, 0]
            dv[:, g] += r1["v"][:, 0]
            np.testing.assert_allclose(full["q"][:, h], r1["q"][:, 0], atol=1e-13)
    np.testing.assert_allclose(full["k"], dk, atol=1e-12)
    np.testing.assert_allclose(full["v"], dv, atol=1e-12)


# ----------------------------------------------------------------------------
# 6. scalar brute force on tiny inputs
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("mode", MODES)
def test_brute_force_scalar_loops(mode):
    par, meta = _tiny_params(mode, seed=71)
    p = _build(par, meta)
    O, lse = oracle.forward(p, rounded=False)
    r = oracle.backward(p, O, lse, par["do"], rounded=False)
    G, dqk, dv, sc = p.G, p.d_qk, p.d_v, p.scale
    Kall = par["kv"] if meta["shared"] else par["k"]
    Vall = par["kv"][..., :dv] if meta["shared"] else par["v"]
    dq = np.zeros_like(par["q"])
    dK = np.zeros_like(Kall)
    dV = np.zeros((Kall.shape[0], meta["Hkv"], dv))
    dC = np.zeros_like(par["cmp_kv"]) if "cmp_kv" in par else None
    dsk = np.zeros(p.Hq)
    off = coff = 0
    for b, L in enumerate(meta["lens"]):
        for t in range(L):
            tq = off + t
            for g in range(meta["Hkv"]):
                counts, ccounts = _selection_counts(meta, tq, g, b, t, L, off)
                keys = []                                     # (kind, global row), with multiplicity
                for rr in range(L):
                    keys += [("o", off + rr)] * int(counts[rr])
                if ccounts is not None:
                    for c in range(len(ccounts)):
                        keys += [("c", coff + c)] * int(ccounts[c])
                for j in range(G):
                    h = g * G + j
                    s = []
                    for kind, row in keys:
                        kr = Kall[row, g] if kind == "o" else par["cmp_kv"][row, g]
                        s.append(sc * sum(par["q"][tq, h, i] * kr[i] for i in range(dqk)))
                    sink = par["sinks"][h] if "sinks" in par else None
                    if not keys and sink is None:
                        assert math.isinf(lse[tq, h]) and np.all(O[tq, h] == 0)
                        continue
                    mx = max(s + ([sink] if sink is not None else []))
                    z = sum(math.exp(x - mx) for x in s) + (math.exp(sink - mx) if sink is not None else 0)
                    l = mx + math.log(z)
                    assert abs(l - lse[tq, h]) < 1e-12
                    P = [math.exp(x - l) for x in s]
                    vrows = [(Vall[row, g] if kind == "o" else par["cmp_kv"][row, g][:dv]) for kind, row in keys]
                    o = [sum(P[n] * vrows[n][c] for n in range(len(keys))) for c in range(dv)]
                    assert max(abs(o[c] - O[tq, h, c]) for c in range(dv)) < 1e-12
                    do = par["do"][tq, h]
                    delta = sum(do[c] * o[c] for c in range(dv))
                    dP = [sum(do[c] * vrows[n][c] for c in range(dv)) for n in range(len(keys))]
                    dS = [P[n] * (dP[n] - delta) for n in range(len(keys))]
                    for n, (kind, row) in enumerate(keys):
                        kr = Kall[row, g] if kind == "o" else par["cmp_kv"][row, g]
                        for i in range(dqk):
                            dq[tq, h, i] += sc * dS[n] * kr[i]
                            if kind == "o":
                                dK[row, g, i] += sc * dS[n] * par["q"][tq, h, i]
                            else:
                                dC[row, g, i] += sc * dS[n] * par["q"][tq, h, i]
                        for c in range(dv):
                            if kind == "o":
                                dV[row, g, c] += P[n] * do[c]
                            else:
                                dC[row, g, c] += P[n] * do[c]
                    if sink is not None:
                        dsk[h] += -math.exp(sink - l) * sum(P[n] * dP[n] for n in range(len(keys)))
        off += L
        if "cmp_lens" in meta:
            coff += meta["cmp_lens"][b]
    np.testing.assert_allclose(r["dq"], dq, atol=1e-12)
    if meta["shared"]:
        dK[..., :dv] += dV
        np.testing.assert_allclose(r["dkv"], dK, atol=1e-12)
    else:
        np.testing.assert_allclose(r["dk"], dK, atol=1e-12)
        np.testing.assert_allclose(r["dv"], dV, atol=1e-12)
    if dC is not None:
        np.testing.assert_allclose(r["dcmp"], dC, atol=1e-12)
    if "sinks" in par:
        np.testing.assert_allclose(r["dsinks"], dsk, atol=1e-12)


# ----------------------------------------------------------------------------
# 7. conversions
# ----------------------------------------------------------------------------

def test_widen_bf16_exact():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000, 0x7F80, 0x0001], dtype=np.uint16)
    x = oracle.widen_bf16(bits)
    assert x[0] == 1.0 and x[1] == -2.0 and x[2] == 1.0 + 2.0 ** -7
    assert x[3] == 0.0 and np.signbit(x[4]) and np.isinf(x[5]) and x[6] == 2.0 ** -133


def test_round_to_bf16_matches_torch_and_ties():
    rng = np.random.default_rng(0)
    x32 = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                          (rng.standard_normal(2000) * 1e-38).astype(np.float32),
                          (rng.standard_normal(2000) * 1e30).astype(np.float32)])
    ours = oracle.round_to_bf16_bits(x32.astype(np.float64))
    ref = torch.tensor(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    ties = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 2.0 ** -8 * 3])
    got = oracle.widen_bf16(oracle.round_to_bf16_bits(ties))
    np.testing.assert_array_equal(got, [1.0, 1 + 2.0 ** -6, -1.0, 3 * 2.0 ** -8])
    # a float64 just above a bf16 tie rounds up, where float32 double rounding would not
    x = 1 + 2.0 ** -8 + 2.0 ** -40
    assert oracle.widen_bf16(oracle.round_to_bf16_bits(np.array([x])))[0] == 1 + 2.0 ** -7


def test_cfa_equals_scfa_listing_every_compressed_row():
    """CFA (every compressed row, no indices) is SCFA whose cmp index list names every
    compressed row of the sequence in order: same rows, same order, same results."""
    par, meta = _tiny_params("cfa", seed=81)
    p_cfa = _build(par, meta)
    Cmax = max(meta["cmp_lens"])
    T = sum(meta["lens"])
    cidx = np.full((T, meta["Hkv"], Cmax), -1, dtype=np.int64)
    off = 0
    for L, C in zip(meta["lens"], meta["cmp_lens"]):
        cidx[off:off + L, :, :C] = np.arange(C)
        off += L
    meta2 = dict(meta, cmp_idx=cidx, cmp_len=np.full((T, meta["Hkv"]), Cmax))
    meta2.pop("cfa")
    p_scfa = _build(par, meta2)
    O1, l1 = oracle.forward(p_cfa, rounded=False)
    O2, l2 = oracle.forward(p_scfa, rounded=False)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(l1, l2)
    r1 = oracle.backward(p_cfa, O1, l1, par["do"], rounded=False)
    r2 = oracle.backward(p_scfa, O2, l2, par["do"], rounded=False)
    for key in r1:
        np.testing.assert_array_equal(r1[key], r2[key])
    # and the compressed rows do take part: some token sees at least one
    assert any(len(oracle.visible_rows(p_cfa, tq, 0)[1]) for tq in range(T))
