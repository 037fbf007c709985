"""Move generator arrays (numpy; bf16 as uint16 bit patterns) to torch tensors."""

from __future__ import annotations

import numpy as np
import torch


def to_torch(inputs: dict, device="cuda") -> dict:
    out = {}
    for k, v in inputs.items():
        if v.dtype == np.uint16:
            t = torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(v))
        out[k] = t.to(device) if device is not None else t
    return out


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """torch bfloat16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def dense_on_device(w, device, seed: int | None = None) -> dict:
    """The workload's dense tensors drawn on the GPU: q, k / kv, v, dO (and cmp_kv)
    as torch bfloat16, with the recipe of ``make_inputs`` -- fp32 N(0, 1) normals
    (dO times the workload's dO scale) rounded to bf16 to nearest even, and
    cmp_kv the float64 mean of each group of cmp_ratio kv rows, rounded the same
    way -- drawn from torch's seeded Philox stream instead of PCG64.  Pair it
    with ``make_inputs(w, dense=False)`` for the sinks and index sets."""
    g = torch.Generator(device=device)
    g.manual_seed(int(w.seed if seed is None else seed))
    lens = w.seq_lengths
    T = sum(lens)
    lead = (w.B, w.S) if w.layout == "BSND" else (T,)

    def normal(shape, mul=1.0):
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if mul != 1.0:
            x.mul_(mul)
        return x.to(torch.bfloat16)

    out = {"q": normal(lead + (w.Hq, w.d_qk))}
    if w.kv_shared:
        out["kv"] = normal(lead + (w.Hkv, w.d_qk))
    else:
        out["k"] = normal(lead + (w.Hkv, w.d_qk))
        out["v"] = normal(lead + (w.Hkv, w.d_v))
    out["do"] = normal(lead + (w.Hq, w.d_v), mul=w.do_scale)
    if w.cmp_topk > 0:
        src = (out["kv"] if w.kv_shared else out["k"]).reshape(T, w.Hkv, w.d_qk)
        parts, start = [], 0
        for L in lens:
            Tc = L // w.cmp_ratio
            seg = src[start:start + Tc * w.cmp_ratio].double().reshape(Tc, w.cmp_ratio, w.Hkv, w.d_qk)
            parts.append(seg.mean(dim=1).float().to(torch.bfloat16))
            start += L
        out["cmp_kv"] = torch.cat(parts, dim=0)
    return out
