"""The five synthetic workloads shaped like the pages' long-sequence cases.

Each workload fixes shapes, selection structure, value distributions and the
seed.  ``scaled`` derives smaller variants with the same structure for tests.

Modes
-----
``block``    block-level selection (NSA style): each index names a block of
             ``block_size`` contiguous KV rows; separate K and V.
``token``    token-level top-k over a shared latent KV head (K = V, MLA style).
``swa_cmp``  sliding-window original KV concatenated with top-k rows of a
             compressed KV (cmp_ratio 4), with per-head fp32 attention sinks.
"""

from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    mode: str                      # "block" | "token" | "swa_cmp"
    layout: str                    # "BSND" | "TND"
    B: int = 1
    S: int = 0                     # BSND sequence length (S_q == S_kv)
    seqlens: tuple = ()            # TND per-sequence lengths (S_q == S_kv per sequence)
    Hq: int = 1
    Hkv: int = 1
    d_qk: int = 64
    d_v: int = 64
    kv_shared: bool = False
    block_size: int = 1
    topk: int = 0                  # slots of ori indices per (token, kv-head); 0 = none
    select: str = "none"           # "diag_uniform" | "zipf" | "token_uniform" | "none"
    cmp_ratio: int = 1
    cmp_topk: int = 0              # slots of cmp indices per (token, kv-head); 0 = none
    cmp_all: bool = False          # compressed KV without indices: every compressed row (CFA)
    used: tuple = ()               # per sequence: tokens that take part (sequsedQ = sequsedOriKv;
                                   # sequsedCmpKv = used // cmp_ratio); () = all
    cmp_len_range: tuple = (0, 0)  # inclusive range of the per-row cmp topk length
    ori_mask: str = "causal"       # "none" | "causal" | "band"
    cmp_mask: str = "causal"       # "none" | "causal"
    win_left: int = 0
    win_right: int = 0
    sinks: bool = False
    zipf_s: float = 0.0
    p_drop: float = 0.0
    do_scale: float = 1.0
    scale: float = 1.0
    seed: int = 0
    notes: str = field(default="", compare=False)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def seq_lengths(self) -> tuple:
        if self.layout == "TND":
            return tuple(self.seqlens)
        return tuple([self.S] * self.B)

    @property
    def T(self) -> int:
        return sum(self.seq_lengths)

    @property
    def n_batches(self) -> int:
        return len(self.seq_lengths)


WORKLOADS = {
    "cfg1_tiny_block_gqa": Workload(
        name="cfg1_tiny_block_gqa", mode="block", layout="BSND", B=1, S=1024,
        Hq=4, Hkv=1, d_qk=64, d_v=64, block_size=64, topk=4, select="diag_uniform",
        scale=1.0 / math.sqrt(64), seed=1001,
        notes="diag block + 3 distinct earlier blocks per token"),
    "cfg2_nsa_g16": Workload(
        name="cfg2_nsa_g16", mode="block", layout="BSND", B=2, S=8192,
        Hq=64, Hkv=4, d_qk=192, d_v=128, block_size=64, topk=16, select="diag_uniform",
        scale=1.0 / math.sqrt(192), seed=1002,
        notes="diag block + 15 distinct uniform earlier blocks per (token, kv-head)"),
    "cfg3_mla_token_topk": Workload(
        name="cfg3_mla_token_topk", mode="token", layout="BSND", B=1, S=32768,
        Hq=128, Hkv=1, d_qk=576, d_v=512, kv_shared=True, block_size=1, topk=2048,
        select="token_uniform", scale=1.0 / math.sqrt(576), seed=1003,
        notes="2048 distinct tokens in [0, t] per token, -1 padded"),
    "cfg4_swa_cmp_sinks": Workload(
        name="cfg4_swa_cmp_sinks", mode="swa_cmp", layout="TND",
        seqlens=(1024, 3000, 8192, 20000), Hq=64, Hkv=1, d_qk=576, d_v=512,
        kv_shared=True, block_size=1, topk=0, select="none", cmp_ratio=4,
        cmp_topk=512, cmp_len_range=(256, 512), ori_mask="band", cmp_mask="causal",
        win_left=127, win_right=0, sinks=True, scale=1.0 / math.sqrt(576), seed=1004,
        notes="SWA 127/0 over ori KV + top-512 of mean-pooled cmp KV, fp32 sinks"),
    "cfg5_zipf_contention": Workload(
        name="cfg5_zipf_contention", mode="block", layout="BSND", B=1, S=65536,
        Hq=64, Hkv=8, d_qk=128, d_v=128, block_size=64, topk=32, select="zipf",
        zipf_s=1.2, p_drop=0.1, do_scale=0.01, scale=1.0 / math.sqrt(128), seed=1005,
        notes="32 distinct blocks in [0, diag] ~ (b+1)^-1.2, 10% dropped, dO x 0.01"),
}

ALIASES = {"cfg1": "cfg1_tiny_block_gqa", "cfg2": "cfg2_nsa_g16",
           "cfg3": "cfg3_mla_token_topk", "cfg4": "cfg4_swa_cmp_sinks",
           "cfg5": "cfg5_zipf_contention"}


def get_workload(name: str) -> Workload:
    return WORKLOADS[ALIASES.get(name, name)]


def scaled(base: Workload | str, suffix: str = "small", **overrides) -> Workload:
    """A smaller variant of ``base`` with the same structure (and its own seed)."""
    if isinstance(base, str):
        base = get_workload(base)
    overrides.setdefault("name", f"{base.name}_{suffix}")
    return dataclasses.replace(base, **overrides)
