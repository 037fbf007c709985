"""Thin PyTorch-facing wrapper over the C ABI.

`SparseAttention` holds the device tensors and attributes of one problem,
marshals them into an `SaArgs`, allocates outputs and workspace with torch
(device memory is PyTorch's job here) and calls `sa_fwd` / `sa_bwd`.  No
arithmetic of the method happens in Python.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

from . import _lib as L


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


_ELEMENT_TYPES = {torch.bfloat16: L.SA_DTYPE_BF16, torch.float16: L.SA_DTYPE_FP16}


def _same_element_type(ref: torch.Tensor, **tensors) -> None:
    """The C ABI takes raw pointers: every 2-byte tensor of a call must hold the
    element type sa_args.dtype names (that of q)."""
    for name, t in tensors.items():
        if t is not None and t.dtype != ref.dtype:
            raise TypeError(f"{name} is {t.dtype}, q is {ref.dtype}: one element type per call")


@dataclass
class SparseAttention:
    layout: str                  # "BSND" | "TND"
    Hq: int
    Hkv: int
    d_qk: int
    d_v: int
    scale: float
    q: torch.Tensor
    k: torch.Tensor | None = None
    v: torch.Tensor | None = None
    kv: torch.Tensor | None = None
    kv_shared: bool = False
    batch: int = 1
    s_q: int = 0
    s_kv: int = 0
    t_q: int = 0
    t_kv: int = 0
    t_cmp: int = 0
    block_size: int = 1
    ori_idx: torch.Tensor | None = None
    ori_topk_len: torch.Tensor | None = None
    cmp_kv: torch.Tensor | None = None
    cmp_idx: torch.Tensor | None = None
    cmp_topk_len: torch.Tensor | None = None
    cmp_ratio: int = 1
    cu_seqlens_q: torch.Tensor | None = None
    cu_seqlens_kv: torch.Tensor | None = None
    cu_seqlens_cmp: torch.Tensor | None = None
    cmp_residual: torch.Tensor | None = None
    sinks: torch.Tensor | None = None
    seqused_q: torch.Tensor | None = None     # [B] int32: query tokens that take part
    seqused_kv: torch.Tensor | None = None    # [B] int32: original KV tokens that take part
    seqused_cmp: torch.Tensor | None = None   # [B] int32: compressed KV rows that take part
    block_table: torch.Tensor | None = None   # [B, max_pages] int32: paged KV cache (k / v / kv are the cache)
    page_size: int = 0
    ori_mask: str = "causal"
    cmp_mask: str = "causal"
    win_left: int = 0
    win_right: int = 0
    flags: int = 0
    _keep: list = field(default_factory=list, repr=False)

    # ---- marshalling -------------------------------------------------------
    @property
    def topk(self) -> int:
        return 0 if self.ori_idx is None else int(self.ori_idx.shape[-1])

    @property
    def cmp_topk(self) -> int:
        return 0 if self.cmp_idx is None else int(self.cmp_idx.shape[-1])

    @property
    def n_tokens(self) -> int:
        return self.batch * self.s_q if self.layout == "BSND" else self.t_q

    def args(self) -> L.SaArgs:
        a = L.SaArgs()
        a.layout_q = L.LAYOUTS[self.layout]
        a.layout_kv = L.LAYOUTS[self.layout]
        if self.q.dtype not in _ELEMENT_TYPES:
            raise TypeError(f"q is {self.q.dtype}: bfloat16 or float16 expected")
        _same_element_type(self.q, k=self.k, v=self.v, kv=self.kv, cmp_kv=self.cmp_kv)
        a.dtype = _ELEMENT_TYPES[self.q.dtype]
        a.batch = self.batch
        a.s_q, a.s_kv = self.s_q, self.s_kv
        a.t_q, a.t_kv, a.t_cmp = self.t_q, self.t_kv, self.t_cmp
        a.n_heads_q, a.n_heads_kv = self.Hq, self.Hkv
        a.d_qk, a.d_v = self.d_qk, self.d_v
        a.kv_shared = 1 if self.kv_shared else 0
        a.block_size = self.block_size
        a.topk, a.cmp_topk = self.topk, self.cmp_topk
        a.cmp_ratio = self.cmp_ratio
        a.ori_mask_mode = L.MASKS[self.ori_mask]
        a.cmp_mask_mode = L.MASKS[self.cmp_mask]
        a.ori_win_left, a.ori_win_right = self.win_left, self.win_right
        a.scale = self.scale
        a.flags = self.flags
        a.q, a.k, a.v, a.kv = _ptr(self.q), _ptr(self.k), _ptr(self.v), _ptr(self.kv)
        a.cmp_kv = _ptr(self.cmp_kv)
        a.ori_idx, a.cmp_idx = _ptr(self.ori_idx), _ptr(self.cmp_idx)
        a.cu_seqlens_q, a.cu_seqlens_kv = _ptr(self.cu_seqlens_q), _ptr(self.cu_seqlens_kv)
        a.cu_seqlens_cmp = _ptr(self.cu_seqlens_cmp)
        a.ori_topk_len, a.cmp_topk_len = _ptr(self.ori_topk_len), _ptr(self.cmp_topk_len)
        a.cmp_residual = _ptr(self.cmp_residual)
        a.sinks = _ptr(self.sinks)
        a.seqused_q, a.seqused_kv = _ptr(self.seqused_q), _ptr(self.seqused_kv)
        a.seqused_cmp = _ptr(self.seqused_cmp)
        a.block_table = _ptr(self.block_table)
        a.page_size = self.page_size
        a.max_pages = 0 if self.block_table is None else int(self.block_table.shape[-1])
        return a

    # ---- allocation helpers ------------------------------------------------
    def _lead(self) -> tuple:
        return (self.batch, self.s_q) if self.layout == "BSND" else (self.t_q,)

    def alloc_fwd(self):
        dev = self.q.device
        o = torch.empty(self._lead() + (self.Hq, self.d_v), dtype=self.q.dtype, device=dev)
        lse = torch.empty(self._lead() + (self.Hq,), dtype=torch.float32, device=dev)
        return o, lse

    def alloc_bwd(self) -> dict:
        dev = self.q.device
        g = {"dq": torch.empty_like(self.q)}
        if self.kv_shared:
            g["dkv"] = torch.empty_like(self.kv)
        else:
            g["dk"], g["dv"] = torch.empty_like(self.k), torch.empty_like(self.v)
        if self.cmp_kv is not None:
            g["dcmp"] = torch.empty_like(self.cmp_kv)
        if self.sinks is not None:
            g["dsinks"] = torch.empty(self.Hq, dtype=torch.float32, device=dev)
        return g

    def fwd_workspace(self) -> torch.Tensor:
        n = L.sa_fwd_get_workspace_size(self.args())
        return torch.empty(max(n, 1), dtype=torch.uint8, device=self.q.device)

    def bwd_workspace(self) -> torch.Tensor:
        n = L.sa_bwd_get_workspace_size(self.args())
        return torch.empty(max(n, 1), dtype=torch.uint8, device=self.q.device)

    # ---- calls -------------------------------------------------------------
    def forward(self, o=None, lse=None, ws=None, stream=None):
        if o is None:
            o, lse = self.alloc_fwd()
        if ws is None:
            ws = self.fwd_workspace()
        _same_element_type(self.q, o=o)
        out = L.SaFwdOut(o=_ptr(o), lse=_ptr(lse))
        st = torch.cuda.current_stream().cuda_stream if stream is None else stream
        L.sa_fwd(self.args(), out, _ptr(ws), ws.numel(), st)
        return o, lse

    def backward(self, o, lse, d_o, grads=None, ws=None, stream=None) -> dict:
        if grads is None:
            grads = self.alloc_bwd()
        if ws is None:
            ws = self.bwd_workspace()
        _same_element_type(self.q, o=o, d_o=d_o, dq=grads["dq"], dk=grads.get("dk"), dv=grads.get("dv"),
                           dkv=grads.get("dkv"), dcmp=grads.get("dcmp"))
        io = L.SaBwdIo(o=_ptr(o), d_o=_ptr(d_o), lse=_ptr(lse), dq=_ptr(grads["dq"]),
                       dk=_ptr(grads.get("dk")), dv=_ptr(grads.get("dv")),
                       dkv=_ptr(grads.get("dkv")), dcmp_kv=_ptr(grads.get("dcmp")),
                       dsinks=_ptr(grads.get("dsinks")))
        st = torch.cuda.current_stream().cuda_stream if stream is None else stream
        L.sa_bwd(self.args(), io, _ptr(ws), ws.numel(), st)
        return grads

    def delta(self, o, d_o, stream=None) -> torch.Tensor:
        _same_element_type(self.q, o=o, d_o=d_o)
        out = torch.empty(self._lead() + (self.Hq,), dtype=torch.float32, device=self.q.device)
        st = torch.cuda.current_stream().cuda_stream if stream is None else stream
        L.sa_softmax_grad_preprocess(self.args(), _ptr(o), _ptr(d_o), _ptr(out), st)
        return out

    def softmax_l1norm(self, lse, ori: bool = True, cmp: bool = True, stream=None):
        """The SoftmaxL1Norm outputs (sa_softmax_l1norm): (ori [.., Hkv, topk] or None,
        cmp [.., Hkv, cmp_topk] or None), fp32, for the index lists this problem has."""
        ori_out = cmp_out = None
        if ori and self.topk > 0:
            ori_out = torch.empty(self._lead() + (self.Hkv, self.topk), dtype=torch.float32, device=self.q.device)
        if cmp and self.cmp_topk > 0 and self.cmp_kv is not None:
            cmp_out = torch.empty(self._lead() + (self.Hkv, self.cmp_topk), dtype=torch.float32, device=self.q.device)
        st = torch.cuda.current_stream().cuda_stream if stream is None else stream
        L.sa_softmax_l1norm(self.args(), _ptr(lse), _ptr(ori_out), _ptr(cmp_out), st)
        return ori_out, cmp_out

    def debug_resolve(self, max_rows: int, stream=None):
        n_units = self.n_tokens * self.Hkv
        rows = torch.full((n_units, max(max_rows, 1)), -1, dtype=torch.int32, device=self.q.device)
        counts = torch.zeros(n_units, dtype=torch.int32, device=self.q.device)
        st = torch.cuda.current_stream().cuda_stream if stream is None else stream
        L.sa_debug_resolve(self.args(), _ptr(rows), _ptr(counts), max_rows, st)
        return rows, counts

    def block_index(self, view: int, max_records: int | None = None, stream=None):
        """Records {unit, block, lo, hi} of the block-level index sets as the block
        kernels build them (sa_debug_block_index); returns an int32 [n, 4] device tensor."""
        if max_records is None:
            max_records = self.n_tokens * self.Hkv * max(self.topk, 1)
        rec = torch.full((max(max_records, 1), 4), -1, dtype=torch.int32, device=self.q.device)
        n = torch.zeros(1, dtype=torch.int32, device=self.q.device)
        ws = self.bwd_workspace() if view == L.SA_INDEX_VIEW_KEY_LISTS else None
        st = torch.cuda.current_stream().cuda_stream if stream is None else stream
        L.sa_debug_block_index(self.args(), view, _ptr(ws), 0 if ws is None else ws.numel(), _ptr(rec),
                               max_records, _ptr(n), st)
        count = int(n.item())
        if count > max_records:
            raise RuntimeError(f"{count} records, room for {max_records}")
        return rec[:count]

    def plan(self) -> tuple:
        """(forward kernel, backward kernel) that sa_fwd / sa_bwd run (SA_KERNEL_*)."""
        return L.sa_plan(self.args())

    @staticmethod
    def read_status(ws: torch.Tensor, stream=None) -> int:
        """The status word of a workspace after its last call, as an sa_status."""
        st = torch.cuda.current_stream().cuda_stream if stream is None else stream
        return L.sa_read_status(_ptr(ws), ws.numel(), st)

    # ---- construction from a workload description ---------------------------
    @classmethod
    def from_workload(cls, w, t: dict, flags: int = 0) -> "SparseAttention":
        """``w``: an object with the workload attributes (see gen.configs.Workload);
        ``t``: device tensors keyed like the generator's arrays (bf16 as torch.bfloat16)."""
        kw = dict(layout=w.layout, Hq=w.Hq, Hkv=w.Hkv, d_qk=w.d_qk, d_v=w.d_v, scale=w.scale,
                  q=t["q"], kv_shared=w.kv_shared, block_size=w.block_size,
                  cmp_ratio=w.cmp_ratio, ori_mask=w.ori_mask, cmp_mask=w.cmp_mask,
                  win_left=w.win_left, win_right=w.win_right, flags=flags)
        if w.kv_shared:
            kw["kv"] = t["kv"]
        else:
            kw["k"], kw["v"] = t["k"], t["v"]
        for key in ("ori_idx", "ori_topk_len", "cmp_kv", "cmp_idx", "cmp_topk_len",
                    "cu_seqlens_q", "cu_seqlens_kv", "cu_seqlens_cmp", "cmp_residual", "sinks",
                    "seqused_q", "seqused_kv", "seqused_cmp"):
            if key in t:
                kw[key] = t[key]
        if w.layout == "BSND":
            kw.update(batch=w.B, s_q=w.S, s_kv=w.S)
        else:
            T = sum(w.seqlens)
            kw.update(batch=len(w.seqlens), t_q=T, t_kv=T,
                      t_cmp=int(t["cmp_kv"].shape[0]) if "cmp_kv" in t else 0)
        return cls(**kw)


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def indexer_kl_grad(q, k, w, idx, p, *, topk_len=None, cu_seqlens_q=None, cu_seqlens_kv=None, batch=None,
                    stream=None):
    """The lightning indexer's KL-loss backward (sa_indexer_kl_grad).

    BSND: q [B, S, H, d], k [B, S_kv, d], w [B, S, H], idx / p [B, S, topk], topk_len
    [B, S] (optional).  TND: the same without B (token-major) plus cu_seqlens_q / _kv.
    Returns (loss per token fp32, dq bf16 like q, dk bf16 like k, dw fp32 like w)."""
    tnd = cu_seqlens_q is not None
    a = L.SaIndexerArgs()
    a.layout = L.SA_LAYOUT_TND if tnd else L.SA_LAYOUT_BSND
    if tnd:
        a.batch = int(cu_seqlens_q.numel()) - 1 if batch is None else batch
        a.t_q, a.t_kv = int(q.shape[0]), int(k.shape[0])
    else:
        a.batch, a.s_q, a.s_kv = int(q.shape[0]), int(q.shape[1]), int(k.shape[1])
    a.n_heads, a.d, a.topk = int(q.shape[-2]), int(q.shape[-1]), int(idx.shape[-1])
    a.q, a.k, a.w, a.idx, a.p = _ptr(q), _ptr(k), _ptr(w), _ptr(idx), _ptr(p)
    a.topk_len = _ptr(topk_len)
    a.cu_seqlens_q, a.cu_seqlens_kv = _ptr(cu_seqlens_q), _ptr(cu_seqlens_kv)
    loss = torch.empty(q.shape[:-2], dtype=torch.float32, device=q.device)
    dq, dk = torch.empty_like(q), torch.empty_like(k)
    dw = torch.empty_like(w)
    g = L.SaIndexerGrads(loss=_ptr(loss), dq=_ptr(dq), dk=_ptr(dk), dw=_ptr(dw))
    n = L.sa_indexer_kl_grad_get_workspace_size(a)
    ws = torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)
    st = torch.cuda.current_stream().cuda_stream if stream is None else stream
    L.sa_indexer_kl_grad(a, g, _ptr(ws), n, st)
    return loss, dq, dk, dw
