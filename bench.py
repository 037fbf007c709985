#!/usr/bin/env python
"""Benchmark of top-k index-selected sparse attention on B200.

One step = the whole hot path on one batch: forward (O, lse) then backward
(rowsum(dO o O), the fused backward, finalize) through the C ABI.  Prints ONE
JSON line (rank 0): the backward TFLOP/s counted over selected, visible
(row, head, key) triples, the roofline fraction of the dominant kernel, the
forward TFLOP/s, an end-to-end figure with host buffers, and the float64
oracle timed on the host cores as a CPU baseline.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       [--workload cfg2] [--no-cpu-baseline] [--no-e2e]
For N > 1 launch under torchrun; every rank runs an independent replica of the
workload (the path has no exchange step), timing is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gen import get_workload, make_inputs  # noqa: E402

METRIC = "sparse-attn bwd TFLOP/s (selected-KV FLOPs) and % of roofline; fwd TFLOP/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------
# workload accounting (host side, from the index tensors)
# ----------------------------------------------------------------------------

def count_work(w, inputs) -> dict:
    """Visible (row, key) pairs per unit and the bytes the selection names.

    visible  -- keys that survive selection, topk lengths and masks (FLOP count)
    gathered -- rows the selection names before masking (block rows clipped to
                the sequence, one row per token / compressed index, the window)
    """
    lens = list(w.seq_lengths)
    T = w.T
    vis = np.zeros((T, w.Hkv), dtype=np.int64)
    gat = np.zeros((T, w.Hkv), dtype=np.int64)
    npair = np.zeros((T, w.Hkv), dtype=np.int64)   # (token, kv-head, usable block slot) with a visible row
    start = 0
    for L in lens:
        t = np.arange(L)[:, None, None]
        ta = t  # equal query / key lengths
        if w.topk:
            idx = inputs["ori_idx"].reshape(T, w.Hkv, -1)[start:start + L].astype(np.int64)
            slot = np.arange(idx.shape[2])[None, None, :]
            ok = idx >= 0
            if "ori_topk_len" in inputs:
                ok &= slot < inputs["ori_topk_len"].reshape(T, w.Hkv)[start:start + L, :, None]
            if w.block_size > 1:
                first = idx * w.block_size
                ok &= first < L
                last = np.minimum(first + w.block_size, L) - 1
                lo, hi = first, last
                if w.ori_mask == "causal":
                    hi = np.minimum(hi, ta)
                elif w.ori_mask == "band":
                    lo = np.maximum(lo, ta - w.win_left)
                    hi = np.minimum(hi, ta + w.win_right)
                v = np.where(ok, np.maximum(hi - lo + 1, 0), 0)
                g = np.where(ok, last - first + 1, 0)
                npair[start:start + L] += (v > 0).sum(-1)
            else:
                ok &= idx < L
                m = ok.copy()
                if w.ori_mask == "causal":
                    m &= idx <= ta
                elif w.ori_mask == "band":
                    m &= (idx >= ta - w.win_left) & (idx <= ta + w.win_right)
                v, g = m, ok
            vis[start:start + L] += v.sum(-1)
            gat[start:start + L] += g.sum(-1)
        else:
            tt = np.arange(L)
            lo, hi = np.zeros(L, dtype=np.int64), np.full(L, L - 1)
            if w.ori_mask == "causal":
                hi = np.minimum(hi, tt)
            elif w.ori_mask == "band":
                lo = np.maximum(lo, tt - w.win_left)
                hi = np.minimum(hi, tt + w.win_right)
            n = np.maximum(hi - lo + 1, 0)[:, None]
            vis[start:start + L] += n
            gat[start:start + L] += n
        if w.cmp_topk:
            cidx = inputs["cmp_idx"].reshape(T, w.Hkv, -1)[start:start + L].astype(np.int64)
            slot = np.arange(cidx.shape[2])[None, None, :]
            ok = (cidx >= 0) & (cidx < L // w.cmp_ratio)
            if "cmp_topk_len" in inputs:
                ok &= slot < inputs["cmp_topk_len"].reshape(T, w.Hkv)[start:start + L, :, None]
            m = ok & ((cidx + 1) * w.cmp_ratio - 1 <= ta)
            vis[start:start + L] += m.sum(-1)
            gat[start:start + L] += ok.sum(-1)
        start += L
    G = w.G
    triples = int(vis.sum()) * G
    n_pairs = int(npair.sum())
    row_bytes = (w.d_qk + (0 if w.kv_shared else w.d_v)) * 2
    gathered = int(gat.sum()) * row_bytes
    Tk = T
    n_q, n_v = T * w.Hq * w.d_qk * 2, T * w.Hq * w.d_v * 2
    lse_b = T * w.Hq * 4
    kv_out = Tk * w.Hkv * (w.d_qk + (0 if w.kv_shared else w.d_v)) * 2
    if w.cmp_topk:
        kv_out += sum(L // w.cmp_ratio for L in lens) * w.Hkv * w.d_qk * 2
    return {
        "triples": triples,
        "fwd_flops": 2 * (w.d_qk + w.d_v) * triples,
        "bwd_flops": 2 * (3 * w.d_qk + 2 * w.d_v) * triples,
        "gathered_bytes": gathered,
        # forward kernel: gathered rows + read Q + write O, lse
        "fwd_bytes": gathered + n_q + n_v + lse_b,
        # fused backward kernel: gathered rows + read Q, dO, lse, Delta + write dQ + dK/dV once
        "bwd_main_bytes": gathered + n_q + n_v + 2 * lse_b + n_q + kv_out,
        # key-stationary dK/dV kernel: S, dP, dV, dK contractions; streams each selecting
        # token's G query and dO rows once per (token, slot) plus the KV blocks once
        "kv_flops": 4 * (w.d_qk + w.d_v) * triples,
        "kv_bytes": n_pairs * w.G * (w.d_qk + w.d_v) * 2 + 2 * n_pairs * w.G * 4 + kv_out + kv_out,
        # ... with dQ formed in the same kernel: + the dQ contraction and the dQ partials
        # (fp32, added once per (token, slot)) read-modify-written through L2
        "kvq_flops": 2 * (3 * w.d_qk + 2 * w.d_v) * triples,
        "kvq_bytes": n_pairs * w.G * (w.d_qk + w.d_v) * 2 + 2 * n_pairs * w.G * 4 + kv_out + kv_out
                     + T * w.Hq * w.d_qk * 4 * 2,
        # query-stationary dQ pass: S, dP, dQ contractions over the gathered rows
        "dq_flops": 2 * (2 * w.d_qk + w.d_v) * triples,
        "dq_bytes": gathered + n_q + n_v + 2 * lse_b + n_q,
        # fp32 reductions of the fused query-stationary backward: every visible row of
        # every 16-head slice adds its dK/dV (dKV) row
        "red_bytes_qs": int(vis.sum()) * ((G + 15) // 16) * (w.d_qk + (0 if w.kv_shared else w.d_v)) * 4,
        # ... of the token-level tensor-core backward: one dKV row per visible row and 64-head slice
        "red_bytes_tk": int(vis.sum()) * ((G + 63) // 64) * w.d_qk * 4,
        "units": T * w.Hkv,
        "_npair": npair,
    }


def kv_reduction_bytes(w, inputs, work: dict) -> int:
    """fp32 reduction bytes of the key-stationary backward with dQ in the kernel: one
    dQ row per (token, head, selected block with a visible row) and one dK/dV flush
    per work item (a chunk of a block's token list), with the work-item sizing the
    library uses (a model of it: the count is reported, not used for timing)."""
    G = w.G
    rpt = G if G in (1, 2, 4) else (G + 7) // 8 * 8
    tpt = 128 // rpt
    nblk = (w.S + 63) // 64
    n_slots = w.B * w.S * w.Hkv * w.topk
    win = w.S
    fit = (48 << 20) // (w.Hq * w.d_qk * 4) // 64 * 64
    need = 128 * nblk // max(1, w.topk)
    if 64 <= fit < w.S and fit >= need:
        win = fit
    want = -(-n_slots // 592)
    lo, hi = tpt, (512 // tpt) * tpt
    if want < lo:
        want = -(-n_slots // 148)
    want = min(max(want, lo), hi)
    chunk = -(-want // tpt) * tpt
    idx = inputs["ori_idx"].reshape(w.B, w.S, w.Hkv, -1).astype(np.int64)
    slot = np.arange(idx.shape[3])[None, None, None, :]
    ok = idx >= 0
    if "ori_topk_len" in inputs:
        ok &= slot < inputs["ori_topk_len"].reshape(w.B, w.S, w.Hkv)[..., None]
    ta = np.arange(w.S)[None, :, None, None]
    ok &= idx * 64 < w.S
    if w.ori_mask == "causal":
        ok &= idx * 64 <= ta
    elif w.ori_mask == "band":
        last = np.minimum(idx * 64 + 63, w.S - 1)
        ok &= (idx * 64 <= ta + w.win_right) & (last >= ta - w.win_left)
    bb = np.broadcast_to(np.arange(w.B)[:, None, None, None], idx.shape)
    gg = np.broadcast_to(np.arange(w.Hkv)[None, None, :, None], idx.shape)
    ww = np.broadcast_to(ta // win, idx.shape)
    lists = ((bb * ((w.S + win - 1) // win) + ww) * w.Hkv + gg) * nblk + np.where(ok, idx, 0)
    counts = np.bincount(lists[ok].ravel())
    n_chunks = int((-(-counts // chunk)).sum())
    dq = int(work["_npair"].sum()) * G * w.d_qk * 4
    return dq + n_chunks * 64 * (w.d_qk + w.d_v) * 4


def load_peaks() -> tuple:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches this build."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        data = json.load(f)
    ent = data.get(f"{kernel}@{workload}")
    if not ent:
        return None
    if ent.get("source_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "top_sparse_attention_attn_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh", ".h")):
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


# ----------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self) -> dict:
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# the CPU baseline: the float64 oracle on a bounded sample of units
# ----------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_baseline(w, inputs, budget_s: float = 12.0, seed: int = 0) -> dict:
    """Time the oracle's backward on random units of the workload (forward for the
    same units computed first, untimed)."""
    import oracle  # the CPU baseline leg is the one place the benchmark runs the oracle
    p = oracle.Problem.from_inputs(w, inputs)
    rng = np.random.default_rng(seed)
    do = inputs["do"].reshape(w.T, w.Hq, w.d_v)
    flops = 0
    elapsed = 0.0
    n_units = 0
    G = w.G
    while elapsed < budget_s:
        batch = [(int(rng.integers(w.T)), int(rng.integers(w.Hkv))) for _ in range(32)]
        fw = oracle.forward(p, units=batch)

        class Rows:
            def __init__(self, k):
                self.k = k

            def __getitem__(self, key):
                tq, hs = key
                g = hs.start // G
                return fw[(tq, g)][self.k]

        t0 = time.perf_counter()
        oracle.backward(p, Rows(0), Rows(1), do, units=batch)
        elapsed += time.perf_counter() - t0
        for tq, g in batch:
            flops += oracle.unit_flops(p, tq, g)[1]
        n_units += len(batch)
    return {"value": flops / elapsed / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle", "elapsed_s": elapsed,
            "sample": f"{n_units} random (token, kv-head) units of {w.name}, float64 NumPy backward "
                      f"({elapsed:.1f} s of CPU time)"}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

def workload_of(args):
    """The named workload, optionally with overrides ("S=2048,B=1") for profiling runs."""
    w = get_workload(args.workload)
    ov = getattr(args, "override", None)
    if ov:
        from gen import scaled
        kw = {}
        for item in ov.split(","):
            k, v = item.split("=")
            kw[k.strip()] = type(getattr(w, k.strip()))(v)
        w = scaled(w, "override", **kw)
    return w


def max_over_ranks(values, world: int, device=None) -> list:
    """Element-wise max of per-rank timings (every rank gets the result)."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def aggregate_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank / (max_ms * 1e-3)


KERNEL_NAMES = {
    1: "qb_kernel (query-stationary block forward, TMA-fed, mma.sync tiles)",
    2: "tk_fwd_kernel (token-level tcgen05 forward)",
    3: "fwd_kernel (generic forward)",
    4: "kv_bwd_kernel (key-stationary dK/dV/dQ, dQ by fp32 atomics)",
    5: "kv_bwd_kernel (key-stationary dK/dV) + qb_kernel<dQ> pass",
    6: "tk_bwd_kernel (token-level tcgen05 backward)",
    7: "bwd_kernel (generic fused backward)",
    8: "bq_fwd_kernel (block forward on tcgen05)",
}


def compulsory_bytes(w, work) -> dict:
    """Bytes any implementation moves at least once: the forward reads Q and K/V (or
    the shared KV and cmp_kv) and writes O and lse; the backward reads Q, K/V, dO, O
    and lse and writes dQ and dK/dV (dKV, dCmpKv) in bf16."""
    T = w.T
    q = T * w.Hq * w.d_qk * 2
    o = T * w.Hq * w.d_v * 2
    lse = T * w.Hq * 4
    kv = T * w.Hkv * (w.d_qk + (0 if w.kv_shared else w.d_v)) * 2
    if w.cmp_topk:
        kv += sum(L // w.cmp_ratio for L in w.seq_lengths) * w.Hkv * w.d_qk * 2
    return {"fwd": q + kv + o + lse, "bwd": q + kv + 2 * o + lse + q + kv}


def fractions(work, comp, peaks, fwd_ms, bwd_ms) -> dict:
    """Roofline fractions (burst tensor peak, measured HBM bandwidth):
    gather_model -- the slower of FLOPs at the tensor peak and gathered + compulsory
                    bytes at HBM bandwidth, over the measured time;
    tensor       -- the slower of FLOPs at the tensor peak and compulsory bytes only
                    (the stricter figure: gathers that hit L2 or are avoided do not count).
    A fraction above 1 means that model does not bind (the kernel beat it)."""
    P, BW = peaks["bf16_tflops"] * 1e12, peaks["hbm_gbs"] * 1e9
    out = {}
    for side, ms, flops, gbytes in (("fwd", fwd_ms, work["fwd_flops"], work["fwd_bytes"]),
                                    ("bwd", bwd_ms, work["bwd_flops"], work["bwd_main_bytes"])):
        ns = max(flops / P, gbytes / BW) * 1e3 / ms
        tc = max(flops / P, comp[side] / BW) * 1e3 / ms
        out[f"{side}_gather_model_frac"] = ns
        out[f"{side}_tensor_frac"] = tc
        out[f"{side}_gather_model_binding"] = ns <= 1.0
    return out


def setup_problem(w, dev, flags: int, host_dense: bool):
    """Inputs, accounting and the SparseAttention object of one workload.  The index
    sets come from the NumPy generator; the dense tensors from the GPU generator
    (same recipe, torch's Philox stream) unless host_dense asks for the NumPy ones."""
    from gen.torch_io import dense_on_device, to_torch
    from top_sparse_attention_attn_b200 import SparseAttention
    inputs = make_inputs(w, dense=host_dense)
    work = count_work(w, inputs)
    t = to_torch(inputs, dev)
    if not host_dense:
        t.update(dense_on_device(w, dev))
    return SparseAttention.from_workload(w, t, flags=flags), t, inputs, work


def measure(sa, t, K: int, warmup: int, use_graph: bool, flush, stream, world: int, hook_passes=True) -> dict:
    """Forward and backward times of one problem: K steps, L2 flushed before each,
    CUDA events on the launching stream.  With graphs the timed steps replay a graph
    of each call; a third graph holds the whole step (forward then backward), whose
    replay time minus the forward's is the backward inside a step."""
    import torch
    from top_sparse_attention_attn_b200 import _lib as L
    o, lse = sa.alloc_fwd()
    grads = sa.alloc_bwd()
    ws_f, ws_b = sa.fwd_workspace(), sa.bwd_workspace()

    def step():
        sa.forward(o, lse, ws_f)
        sa.backward(o, lse, t["do"], grads, ws_b)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    launches_per_step = None
    if use_graph:
        side = torch.cuda.Stream(stream.device)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        g_fwd, g_bwd, g_step = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        n0 = L.sa_kernel_launch_count()
        with torch.cuda.graph(g_fwd):
            sa.forward(o, lse, ws_f)
        with torch.cuda.graph(g_bwd):
            sa.backward(o, lse, t["do"], grads, ws_b)
        launches_per_step = L.sa_kernel_launch_count() - n0
        with torch.cuda.graph(g_step):
            step()
        for _ in range(2):
            g_fwd.replay()
            g_bwd.replay()
            g_step.replay()
        torch.cuda.synchronize()

    def timed_pass(which):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
        for e in ev:  # materialise the raw cudaEvent_t handles
            for x in e:
                x.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        for k in range(K):
            flush.zero_()                          # L2 flushed between timed steps
            e0, e1, e2, mb, me = ev[k]
            e0.record(stream)
            if which is None and use_graph:
                g_fwd.replay()
                e1.record(stream)
                g_bwd.replay()
            else:
                if which == L.TIME_FWD:
                    L.sa_set_timing_events(mb.cuda_event, me.cuda_event, which)
                sa.forward(o, lse, ws_f)
                L.sa_set_timing_events(None, None, -1)
                e1.record(stream)
                if which is not None and which != L.TIME_FWD:
                    L.sa_set_timing_events(mb.cuda_event, me.cuda_event, which)
                sa.backward(o, lse, t["do"], grads, ws_b)
                L.sa_set_timing_events(None, None, -1)
            e2.record(stream)
        torch.cuda.synchronize()
        fwd = sum(e[0].elapsed_time(e[1]) for e in ev) / K
        bwd = sum(e[1].elapsed_time(e[2]) for e in ev) / K
        kern = sum(e[3].elapsed_time(e[4]) for e in ev) / K if which is not None else 0.0
        return fwd, bwd, kern

    def step_graph_pass():
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        torch.cuda.synchronize()
        for k in range(K):
            flush.zero_()
            ev[k][0].record(stream)
            g_step.replay()
            ev[k][1].record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in ev) / K

    r = {}
    n0 = L.sa_kernel_launch_count()
    r["fwd_ms"], r["bwd_ms"], _ = timed_pass(None)
    r["launches"] = launches_per_step * K if use_graph else L.sa_kernel_launch_count() - n0
    r["step_graph_ms"] = step_graph_pass() if use_graph else r["fwd_ms"] + r["bwd_ms"]
    r["bwd_in_step_ms"] = max(r["step_graph_ms"] - r["fwd_ms"], 1e-6)
    if hook_passes:
        # attribution passes (eager calls, not part of the timed steps): the timing hook
        # around the backward's main kernel, the separate dQ pass, the forward kernel
        r["fwd_eager_ms"], r["bwd_eager_ms"], r["bwd_kernel_ms"] = timed_pass(L.TIME_BWD_KV)
        r["dq_kernel_ms"] = timed_pass(L.TIME_BWD_DQ)[2]
        r["fwd_kernel_ms"] = timed_pass(L.TIME_FWD)[2]
    r["_bufs"] = (o, lse, grads, ws_f, ws_b)
    return r


def dominant_kernel_roofline(w, work, comp, peaks, peak_src, plan, m) -> dict:
    """Roofline of the longest kernel: its FLOPs at the burst tensor peak against its
    compulsory bytes at HBM bandwidth (whichever is slower sets the bound), over its
    CUDA-event time; plus the spec fraction of the same kernel and the DRAM
    bytes of its committed ncu capture (null when the sources changed since)."""
    fwd_k, bwd_k = plan
    cands = [(KERNEL_NAMES[bwd_k], m.get("bwd_kernel_ms", 0.0), "bwd"),
             (KERNEL_NAMES[fwd_k], m.get("fwd_kernel_ms", 0.0), "fwd")]
    if m.get("dq_kernel_ms"):
        cands.append(("qb_kernel<dQ> (query-stationary dQ pass)", m["dq_kernel_ms"], "bwd"))
    name, kms, side = max(cands, key=lambda c: c[1])
    if side == "bwd" and bwd_k == 5:  # split backward: each kernel carries its own contractions
        flops = work["dq_flops"] if name.startswith("qb_kernel") else work["kv_flops"]
    else:
        flops = work[f"{side}_flops"]
    cbytes = comp[side]
    gbytes = work["fwd_bytes"] if side == "fwd" else work["bwd_main_bytes"]
    P, BW = peaks["bf16_tflops"] * 1e12, peaks["hbm_gbs"] * 1e9
    t_f, t_b = flops / P, cbytes / BW
    bound = "tensor" if t_f >= t_b else "hbm"
    if bound == "tensor":
        achieved, peak, unit = flops / (kms * 1e-3) / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    else:
        achieved, peak, unit = cbytes / (kms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s"
    traffic = load_traffic(name.split(" ")[0], w.name)
    ns = max(t_f, gbytes / BW) * 1e3 / kms
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
            "traffic": traffic, "kernel": name, "kernel_ms": kms,
            "algorithmic_flops": flops, "algorithmic_bytes": cbytes,
            "peak_source": ("measured MEASURED_PEAKS.json (bf16 burst; HBM copy)" if peak_src == "measured"
                            else "fallback"),
            "t_roof_ms": max(t_f, t_b) * 1e3,
            "gather_model_frac": ns, "gather_model_binding": ns <= 1.0,
            "dram_over_compulsory": None if traffic is None else traffic / cbytes}


def config_of(w, work, world: int, flags: str) -> dict:
    return {"workload": w.name, "B": w.B, "S": w.S, "Hq": w.Hq, "Hkv": w.Hkv,
            "d_qk": w.d_qk, "d_v": w.d_v, "block_size": w.block_size, "topk": w.topk,
            "parallelism": f"replicas{world}", "flags": flags or "default",
            "visible_triples": work["triples"], "gathered_bytes": work["gathered_bytes"]}


PER_WORKLOAD = (("cfg1", 20), ("cfg5", 5), ("cfg4", 5), ("cfg3", 3))


def run_ours(args, rank: int, world: int, local_rank: int) -> dict | None:
    import torch
    from top_sparse_attention_attn_b200 import _lib as L

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workload_of(args)
    flags = 0
    for f in filter(None, args.flags.split(",")):
        flags |= {"dq_separate": L.SA_FLAG_DQ_SEPARATE, "query_stationary": L.SA_FLAG_QUERY_STATIONARY_BWD,
                  "fwd_block_tc": L.SA_FLAG_FWD_BLOCK_TC, "token_fwd_unpaired": L.SA_FLAG_TOKEN_FWD_UNPAIRED}[f]
    sa, t, inputs, work = setup_problem(w, dev, flags, host_dense=False)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    use_graph = not args.no_graph
    K = args.steps
    plan = sa.plan()

    with ClockSampler(local_rank) as clk:
        m = measure(sa, t, K, args.warmup, use_graph, flush, stream, world)
    keys = ["fwd_ms", "bwd_ms", "bwd_kernel_ms", "dq_kernel_ms", "fwd_kernel_ms", "fwd_eager_ms",
            "bwd_eager_ms", "step_graph_ms"]
    for k_, v in zip(keys, max_over_ranks([m[k_] for k_ in keys], world, dev)):
        m[k_] = v
    m["bwd_in_step_ms"] = max(m["step_graph_ms"] - m["fwd_ms"], 1e-6)
    o, lse, grads, ws_f, ws_b = m.pop("_bufs")
    step_ms = m["fwd_ms"] + m["bwd_ms"]

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        host_in = {k: v.cpu().pin_memory() for k, v in t.items()}
        host_out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in grads.items()}
        h2d = sum(v.numel() * v.element_size() for v in host_in.values())
        d2h = sum(v.numel() * v.element_size() for v in host_out.values())

        def e2e_step():
            for k_, v in host_in.items():
                t[k_].copy_(v, non_blocking=True)
            sa.forward(o, lse, ws_f)
            sa.backward(o, lse, t["do"], grads, ws_b)
            for k_, v in host_out.items():
                v.copy_(grads[k_], non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        es = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for k in range(K):
            flush.zero_()
            es[k][0].record(stream)
            e2e_step()
            es[k][1].record(stream)
        torch.cuda.synchronize()
        e2e_ms = torch.tensor([sum(a.elapsed_time(b) for a, b in es) / K], dtype=torch.float64, device=dev)
        if world > 1:
            torch.distributed.all_reduce(e2e_ms, op=torch.distributed.ReduceOp.MAX)
        e2e = {"value": world * work["bwd_flops"] / (e2e_ms.item() * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms.item(),
               "note": "bwd FLOPs over the whole step: H2D of inputs, forward, backward, D2H of gradients"}

    # the other workloads, measured in the same run (every rank runs them: the
    # barriers inside the timed passes stay matched); fewer steps for the long ones
    per_workload = {}
    if not args.no_per_workload and args.override is None:
        for name, k_steps in PER_WORKLOAD:
            w2 = get_workload(name)
            if w2.name == w.name:
                continue
            sa2, t2, _, work2 = setup_problem(w2, dev, 0, host_dense=False)
            with ClockSampler(local_rank) as clk2:
                m2 = measure(sa2, t2, k_steps, 2, use_graph, flush, stream, world)
            m2.pop("_bufs")
            ks = ["fwd_ms", "bwd_ms", "bwd_kernel_ms", "fwd_kernel_ms", "step_graph_ms", "dq_kernel_ms"]
            for k_, v in zip(ks, max_over_ranks([m2[k_] for k_ in ks], world, dev)):
                m2[k_] = v
            m2["bwd_in_step_ms"] = max(m2["step_graph_ms"] - m2["fwd_ms"], 1e-6)
            if rank == 0:
                peaks2, src2 = load_peaks()
                comp2 = compulsory_bytes(w2, work2)
                plan2 = sa2.plan()
                fr = fractions(work2, comp2, peaks2, m2["fwd_ms"], m2["bwd_ms"])
                fr_step = fractions(work2, comp2, peaks2, m2["fwd_ms"], m2["bwd_in_step_ms"])
                roof2 = dominant_kernel_roofline(w2, work2, comp2, peaks2, src2, plan2, m2)
                per_workload[name] = {
                    "workload": w2.name, "steps": k_steps,
                    "fwd_ms": m2["fwd_ms"], "bwd_ms": m2["bwd_ms"], "bwd_in_step_ms": m2["bwd_in_step_ms"],
                    "fwd_tflops": work2["fwd_flops"] / (m2["fwd_ms"] * 1e-3) / 1e12,
                    "bwd_tflops": work2["bwd_flops"] / (m2["bwd_ms"] * 1e-3) / 1e12,
                    "fwd_kernel": KERNEL_NAMES[plan2[0]], "bwd_kernel": KERNEL_NAMES[plan2[1]],
                    **fr,
                    "bwd_gather_model_frac_in_step": fr_step["bwd_gather_model_frac"],
                    "bwd_tensor_frac_in_step": fr_step["bwd_tensor_frac"],
                    "roofline": roof2, "clocks": clk2.summary(),
                    "config": config_of(w2, work2, world, "")}
            del sa2, t2
            torch.cuda.empty_cache()

    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    comp = compulsory_bytes(w, work)
    bwd_tflops = aggregate_rate(work["bwd_flops"], world, m["bwd_ms"]) / 1e12
    fwd_tflops = aggregate_rate(work["fwd_flops"], world, m["fwd_ms"]) / 1e12
    roof = dominant_kernel_roofline(w, work, comp, peaks, peak_src, plan, m)
    fr = fractions(work, comp, peaks, m["fwd_ms"], m["bwd_ms"])
    fr_step = fractions(work, comp, peaks, m["fwd_ms"], m["bwd_in_step_ms"])
    # the fp32 reduction traffic of the backward's main kernel, as achieved GB/s (a
    # reporting model: a failure here must not cost the measurement)
    try:
        if plan[1] == 4:
            red_bytes = kv_reduction_bytes(w, inputs, work)
            red_model = "dQ row per (token, head, block) + dK/dV flush per work item"
        elif plan[1] == 6:
            red_bytes = work["red_bytes_tk"]
            red_model = "dKV row per visible row and 64-head slice"
        elif plan[1] == 7:
            red_bytes = work["red_bytes_qs"]
            red_model = "dK/dV (dKV) row per visible row and 16-head slice"
        else:
            red_bytes, red_model = None, None
    except Exception:  # noqa: BLE001
        red_bytes, red_model = None, None
    line = {
        "metric": METRIC, "value": bwd_tflops, "unit": "TFLOP/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(w, work, world, args.flags),
        "l2": "flushed between timed steps (a 2x L2 write before each)",
        "fwd_tflops": fwd_tflops, "fwd_ms": m["fwd_ms"], "bwd_ms": m["bwd_ms"],
        "timing": "CUDA-graph replays" if use_graph else "eager calls",
        "fwd_eager_ms": m["fwd_eager_ms"], "bwd_eager_ms": m["bwd_eager_ms"],
        "fwd_kernel": KERNEL_NAMES[plan[0]], "bwd_path": KERNEL_NAMES[plan[1]],
        **fr,
        # the backward as part of a one-graph step (forward then backward), minus the
        # forward alone: the fixed cost of starting a graph of its own drops out
        "step_graph_ms": m["step_graph_ms"], "bwd_in_step_ms": m["bwd_in_step_ms"],
        "bwd_gather_model_frac_in_step": fr_step["bwd_gather_model_frac"],
        "bwd_tensor_frac_in_step": fr_step["bwd_tensor_frac"],
        "roofline": roof, "clocks": clk.summary(), "gpu_launches": m["launches"],
        # fp32 dQ / dK / dV reductions (L2 read-modify-writes, not DRAM bytes) of the
        # backward's main kernel, over its measured time
        "reductions": None if red_bytes is None else {
            "bytes": red_bytes, "achieved_gbs": red_bytes / (m["bwd_kernel_ms"] * 1e-3) / 1e9,
            "model": red_model},
        "e2e": e2e,
        "per_workload": per_workload,
    }
    if world == 1 and not args.no_cpu_baseline:
        # the oracle reads the same dense tensors the GPU ran on (host copies of the bits)
        from gen.torch_io import bf16_bits
        for k_ in ("q", "k", "v", "kv", "do", "cmp_kv"):
            if k_ in t:
                inputs[k_] = bf16_bits(t[k_])
        line["cpu_baseline"] = oracle_baseline(w, inputs)
    return line


# ----------------------------------------------------------------------------
# reference arm: the oracle on the host cores
# ----------------------------------------------------------------------------

def run_reference(args, rank: int) -> dict | None:
    if rank != 0:
        return None
    w = workload_of(args)
    inputs = make_inputs(w)
    per_step = getattr(args, "step_budget", None) or max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_baseline(w, inputs, budget_s=1.0, seed=1)
    vals = [oracle_baseline(w, inputs, budget_s=per_step, seed=100 + k) for k in range(args.steps)]
    v = statistics.mean(x["value"] for x in vals)
    work = count_work(w, inputs)
    sample_ms = statistics.mean(x["elapsed_s"] for x in vals) * 1e3
    return {"metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "impl": "reference",
            # each timed step is a bounded sample of the workload's backward (random
            # units); ms_per_step is that measured sample, and a whole backward at the
            # sampled rate is reported beside it
            "ms_per_step": sample_ms,
            "whole_backward_ms_at_sampled_rate": work["bwd_flops"] / (v * 1e12) * 1e3,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, work, 1, ""),
            "l2": "n/a (host cores)",
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": vals[0]["cores"],
                             "kind": "oracle", "sample": vals[0]["sample"]},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="cfg2")
    ap.add_argument("--override", default=None, help="workload overrides for profiling, e.g. S=2048")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager calls instead of CUDA-graph replays")
    ap.add_argument("--no-per-workload", action="store_true", help="skip the other workloads' figures")
    ap.add_argument("--flags", default="", help="kernel variants for measurements: dq_separate | query_stationary | fwd_block_tc | "
                    "token_fwd_unpaired")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        line = run_reference(args, rank)
    else:
        if world > 1:
            import datetime
            import torch
            torch.cuda.set_device(local_rank)
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        line = run_ours(args, rank, world, local_rank)
        if world > 1:
            import torch
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
