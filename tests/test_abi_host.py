"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, its structs match the ctypes mirror, and argument validation returns
the documented status codes without touching a GPU."""

import ctypes
import os
import re
import subprocess
import tempfile

import pytest

from top_sparse_attention_attn_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparse_attn.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(sa_\w+)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert len(names) >= 8
    lib = L.lib()
    for n in names:
        assert hasattr(lib, n), f"{n} declared in sparse_attn.h but not exported"
    assert sorted(L.EXPORTS) == names


def test_abi_version_and_status_strings():
    m = re.search(r"#define SA_ABI_VERSION (\d+)", open(HEADER).read())
    assert L.sa_abi_version() == int(m.group(1))
    for s in range(8):
        assert L.status_string(s).startswith("SA_")
    assert "unknown" in L.status_string(99)


C_PROBE = r"""
#include <stdio.h>
#include <stddef.h>
#include "sparse_attn.h"
#define F(S, m) printf("%s.%s %zu\n", #S, #m, offsetof(S, m));
int main(void) {
  printf("sa_args %zu\nsa_fwd_out %zu\nsa_bwd_io %zu\n", sizeof(sa_args), sizeof(sa_fwd_out), sizeof(sa_bwd_io));
  F(sa_args, layout_kv) F(sa_args, dtype) F(sa_args, ori_win_left) F(sa_args, scale) F(sa_args, flags) F(sa_args, q) F(sa_args, sinks)
  F(sa_args, cmp_idx) F(sa_args, cu_seqlens_cmp) F(sa_bwd_io, dsinks) F(sa_bwd_io, dcmp_kv)
  return 0;
}
"""


def test_struct_layout_matches_header():
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "probe.c")
        exe = os.path.join(d, "probe")
        open(src, "w").write(C_PROBE)
        subprocess.run(["gcc", "-std=c11", "-I", os.path.dirname(HEADER), src, "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    got = dict(line.split() for line in out if line.strip())
    assert int(got["sa_args"]) == ctypes.sizeof(L.SaArgs)
    assert int(got["sa_fwd_out"]) == ctypes.sizeof(L.SaFwdOut)
    assert int(got["sa_bwd_io"]) == ctypes.sizeof(L.SaBwdIo)
    for key, val in got.items():
        if "." in key:
            s, m = key.split(".")
            cls = {"sa_args": L.SaArgs, "sa_bwd_io": L.SaBwdIo}[s]
            assert getattr(cls, m).offset == int(val), key


# ----------------------------------------------------------------------------
# validation (host only: every call below fails before any CUDA call)
# ----------------------------------------------------------------------------

FAKE = 0x10000  # 16-byte aligned, never dereferenced: these calls fail validation first


def _args(**kw):
    a = L.SaArgs()
    a.layout_q = a.layout_kv = L.SA_LAYOUT_BSND
    a.dtype = L.SA_DTYPE_BF16
    a.batch, a.s_q, a.s_kv = 2, 128, 128
    a.n_heads_q, a.n_heads_kv = 16, 4
    a.d_qk, a.d_v = 192, 128
    a.block_size, a.topk = 64, 4
    a.cmp_ratio = 1
    a.ori_mask_mode = L.SA_MASK_CAUSAL
    a.scale = 0.1
    a.q = a.k = a.v = a.ori_idx = FAKE
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def _ws(a):
    n = ctypes.c_size_t(0)
    st = L.lib().sa_bwd_get_workspace_size(ctypes.byref(a), ctypes.byref(n))
    return st, n.value


@pytest.mark.parametrize("kw,status", [
    (dict(), L.SA_OK),
    (dict(n_heads_q=15), L.SA_ERR_PARAM),
    (dict(n_heads_kv=0), L.SA_ERR_PARAM),
    (dict(dtype=L.SA_DTYPE_FP16), L.SA_OK),
    (dict(dtype=7), L.SA_ERR_PARAM),
    (dict(d_qk=96, d_v=96), L.SA_ERR_UNSUPPORTED),
    (dict(d_qk=100), L.SA_ERR_PARAM),
    (dict(d_qk=640), L.SA_ERR_PARAM),
    (dict(block_size=100), L.SA_ERR_PARAM),
    (dict(block_size=0), L.SA_ERR_PARAM),
    (dict(topk=-1), L.SA_ERR_PARAM),
    (dict(q=None), L.SA_ERR_NULLPTR),
    (dict(ori_idx=None), L.SA_ERR_NULLPTR),
    (dict(v=None), L.SA_ERR_NULLPTR),
    (dict(layout_q=5, layout_kv=5), L.SA_ERR_PARAM),
    (dict(layout_kv=5), L.SA_ERR_PARAM),
    (dict(layout_kv=L.SA_LAYOUT_TND), L.SA_ERR_UNSUPPORTED),                 # mixed layouts are not built
    (dict(ori_mask_mode=L.SA_MASK_BAND, ori_win_left=-1), L.SA_ERR_PARAM),
    (dict(cmp_mask_mode=L.SA_MASK_BAND), L.SA_ERR_PARAM),
    (dict(cmp_ratio=0), L.SA_ERR_PARAM),
    (dict(scale=float("nan")), L.SA_ERR_PARAM),
    (dict(cmp_topk=8, cmp_kv=FAKE, cmp_idx=FAKE), L.SA_ERR_UNSUPPORTED),   # compressed KV needs K = V
    (dict(layout_q=L.SA_LAYOUT_TND, layout_kv=L.SA_LAYOUT_TND, t_q=256, t_kv=256), L.SA_ERR_NULLPTR),
    (dict(kv_shared=1, d_qk=128, d_v=128, k=None, v=None), L.SA_ERR_NULLPTR),
    (dict(kv_shared=1, d_qk=128, d_v=128, k=None, v=None, kv=FAKE), L.SA_OK),
    (dict(kv_shared=1, d_qk=128, d_v=256, kv=FAKE), L.SA_ERR_PARAM),
])
def test_validation_codes(kw, status):
    st, _ = _ws(_args(**kw))
    assert st == status, L.status_string(st)
    n = ctypes.c_size_t(0)
    assert L.lib().sa_fwd_get_workspace_size(ctypes.byref(_args(**kw)), ctypes.byref(n)) == status


def test_null_args_and_null_size():
    n = ctypes.c_size_t(0)
    assert L.lib().sa_fwd_get_workspace_size(None, ctypes.byref(n)) == L.SA_ERR_NULLPTR
    assert L.lib().sa_bwd_get_workspace_size(ctypes.byref(_args()), None) == L.SA_ERR_NULLPTR


def _align(x):
    return (x + 255) // 256 * 256


def test_bwd_workspace_size_contract():
    # query-stationary backward: status word, Delta, fp32 dK and dV accumulators
    a = _args(flags=L.SA_FLAG_QUERY_STATIONARY_BWD)
    st, n = _ws(a)
    Tq, Tk = 2 * 128, 2 * 128
    base = 256 + _align(Tq * 16 * 4) + _align(Tk * 4 * 192 * 4) + _align(Tk * 4 * 128 * 4)
    assert st == L.SA_OK and n == base
    # key-stationary backward (block-level, BSND, 64-row blocks): + the inverse index
    # counts, cursor, list offsets, work items (16 B each; a small problem gets
    # chunks of ceil(n_slots / 148) tokens rounded up to whole 128-row tiles), the
    # work count and the entries; a problem this small also takes the bucketed
    # index: per bucket of 512 slots, each list's count and offset, and one flag
    n_lists, n_slots = 2 * 4 * 2, 2 * 128 * 4 * 4
    chunk = -(-(-(-n_slots // 148)) // 16) * 16  # whole tiles of 16 (8 rows per token) or 32 tokens
    max_work = -(-n_slots // chunk) + n_lists
    cells = -(-n_slots // 512) * n_lists
    n_buckets = -(-n_slots // 512)
    index = (2 * _align(4 * n_lists) + _align(4 * (n_lists + 1)) + _align(16 * max_work) + 256
             + _align(4 * n_slots) + 2 * _align(4 * cells) + _align(4 * n_buckets))
    st, n = _ws(_args(flags=L.SA_FLAG_DQ_SEPARATE))
    assert st == L.SA_OK and n == base + index
    # ... + an fp32 dQ accumulator when dQ is formed in the same kernel (the default)
    st, n = _ws(_args())
    assert st == L.SA_OK and n == base + index + _align(Tq * 16 * 192 * 4)
    a = _args(kv_shared=1, d_qk=576, d_v=512, kv=FAKE, n_heads_q=64, n_heads_kv=1, block_size=1,
              layout_q=L.SA_LAYOUT_TND, layout_kv=L.SA_LAYOUT_TND, t_q=1000, t_kv=1000, t_cmp=250, cmp_topk=16, cmp_ratio=4,
              cmp_kv=FAKE, cmp_idx=FAKE, cu_seqlens_q=FAKE, cu_seqlens_kv=FAKE, cu_seqlens_cmp=FAKE)
    st, n = _ws(a)
    expect = 256 + _align(1000 * 64 * 4) + _align(1000 * 576 * 4) + _align(250 * 576 * 4)
    assert st == L.SA_OK and n == expect


def test_calls_fail_before_launch():
    a = _args()
    n = _ws(a)[1]
    io = L.SaBwdIo(o=FAKE, d_o=FAKE, lse=FAKE, dq=FAKE, dk=FAKE, dv=FAKE)
    # workspace too small / missing
    assert L.lib().sa_bwd(ctypes.byref(a), ctypes.byref(io), FAKE, n - 1, None) == L.SA_ERR_WORKSPACE
    assert L.lib().sa_bwd(ctypes.byref(a), ctypes.byref(io), None, n, None) == L.SA_ERR_WORKSPACE
    # missing outputs
    io2 = L.SaBwdIo(o=FAKE, d_o=FAKE, lse=FAKE, dq=FAKE, dk=FAKE)
    assert L.lib().sa_bwd(ctypes.byref(a), ctypes.byref(io2), FAKE, n, None) == L.SA_ERR_NULLPTR
    assert L.lib().sa_bwd(ctypes.byref(a), None, FAKE, n, None) == L.SA_ERR_NULLPTR
    out = L.SaFwdOut(o=FAKE, lse=None)
    assert L.lib().sa_fwd(ctypes.byref(a), ctypes.byref(out), FAKE, 256, None) == L.SA_ERR_NULLPTR
    # misaligned tensor
    out = L.SaFwdOut(o=FAKE, lse=FAKE)
    a.q = FAKE + 2
    assert L.lib().sa_fwd(ctypes.byref(a), ctypes.byref(out), FAKE, 256, None) == L.SA_ERR_PARAM


def test_empty_query_is_a_no_op():
    """An empty query is a successful no-op (aclnnSparseFlashAttentionGrad, Constraints, empty inputs)."""
    a = _args(s_q=0)
    out = L.SaFwdOut(o=None, lse=None)
    assert L.lib().sa_fwd(ctypes.byref(a), ctypes.byref(out), None, 0, None) == L.SA_OK
    io = L.SaBwdIo()
    assert L.lib().sa_bwd(ctypes.byref(a), ctypes.byref(io), None, 0, None) == L.SA_OK
    a = _args(batch=0)
    assert L.lib().sa_fwd(ctypes.byref(a), ctypes.byref(out), None, 0, None) == L.SA_OK
    assert L.lib().sa_softmax_grad_preprocess(ctypes.byref(a), None, None, None, None) == L.SA_OK


def test_no_alloc_rejects_oversized_problem_on_the_host():
    """sa_bwd_no_alloc refuses problems whose workspace exceeds its fixed scratch."""
    cap = L.sa_bwd_no_alloc_max_workspace()
    assert cap >= 1 << 20
    a = _args(batch=8, s_q=8192, s_kv=8192)                 # ~ hundreds of MB of accumulators
    assert _ws(a)[1] > cap
    io = L.SaBwdIo(o=FAKE, d_o=FAKE, lse=FAKE, dq=FAKE, dk=FAKE, dv=FAKE)
    assert L.lib().sa_bwd_no_alloc(ctypes.byref(a), ctypes.byref(io), None) == L.SA_ERR_WORKSPACE
    assert L.lib().sa_bwd_no_alloc(ctypes.byref(_args(n_heads_q=15)), ctypes.byref(io), None) == L.SA_ERR_PARAM


def _plan(a):
    return L.sa_plan(a)


def test_plan_reports_the_kernel_each_problem_gets():
    """sa_plan names the forward / backward kernels sa_fwd / sa_bwd dispatch to."""
    assert _plan(_args()) == (L.SA_KERNEL_FWD_BLOCK, L.SA_KERNEL_BWD_KEY_STATIONARY)
    assert _plan(_args(flags=L.SA_FLAG_DQ_SEPARATE)) == (L.SA_KERNEL_FWD_BLOCK,
                                                         L.SA_KERNEL_BWD_KEY_STATIONARY_DQ_PASS)
    assert _plan(_args(flags=L.SA_FLAG_QUERY_STATIONARY_BWD))[1] == L.SA_KERNEL_BWD_GENERIC
    assert _plan(_args(flags=L.SA_FLAG_FWD_BLOCK_TC)) == (L.SA_KERNEL_FWD_BLOCK_TC, L.SA_KERNEL_BWD_KEY_STATIONARY)
    # the flag touches block problems only
    assert _plan(_args(block_size=16, flags=L.SA_FLAG_FWD_BLOCK_TC))[0] == L.SA_KERNEL_FWD_GENERIC
    # sinks, TND, block sizes other than 64 and unequal lengths leave the key-stationary kernel
    assert _plan(_args(sinks=FAKE))[1] == L.SA_KERNEL_BWD_GENERIC
    assert _plan(_args(block_size=16)) == (L.SA_KERNEL_FWD_GENERIC, L.SA_KERNEL_BWD_GENERIC)
    assert _plan(_args(s_kv=256))[1] == L.SA_KERNEL_BWD_GENERIC
    # token-level shared KV 576 / 512 with 64 heads per kv-head: the tensor-core token kernels
    tok = dict(kv_shared=1, d_qk=576, d_v=512, kv=FAKE, k=None, v=None, n_heads_q=64, n_heads_kv=1,
               block_size=1, topk=32)
    assert _plan(_args(**tok)) == (L.SA_KERNEL_FWD_TOKEN_TC, L.SA_KERNEL_BWD_TOKEN_TC)
    assert _plan(_args(**dict(tok, n_heads_q=16))) == (L.SA_KERNEL_FWD_GENERIC, L.SA_KERNEL_BWD_GENERIC)
    # fp16 inputs run on the generic kernels (the tensor-core kernels take bf16)
    f16 = L.SA_DTYPE_FP16
    assert _plan(_args(dtype=f16)) == (L.SA_KERNEL_FWD_GENERIC, L.SA_KERNEL_BWD_GENERIC)
    assert _plan(_args(**dict(tok, dtype=f16))) == (L.SA_KERNEL_FWD_GENERIC, L.SA_KERNEL_BWD_GENERIC)
    assert _plan(_args(dtype=f16, flags=L.SA_FLAG_FWD_BLOCK_TC))[0] == L.SA_KERNEL_FWD_GENERIC
    with pytest.raises(L.SaError):
        _plan(_args(n_heads_q=15))


def test_dq_separate_is_ignored_past_the_block_kernels_slot_limit():
    """The separate dQ pass holds at most 256 usable slots per unit: with more, the flag is
    ignored (the key-stationary kernel forms dQ), in the plan and in the workspace."""
    a = _args(topk=300, batch=1, s_q=65536, s_kv=65536)
    b = _args(topk=300, batch=1, s_q=65536, s_kv=65536, flags=L.SA_FLAG_DQ_SEPARATE)
    assert _plan(b) == (L.SA_KERNEL_FWD_GENERIC, L.SA_KERNEL_BWD_KEY_STATIONARY)
    assert _ws(a) == _ws(b)


def test_indexer_kl_grad_validates_on_the_host():
    a = L.SaIndexerArgs()
    a.layout, a.batch, a.s_q, a.s_kv = L.SA_LAYOUT_BSND, 2, 64, 64
    a.n_heads, a.d, a.topk = 64, 128, 32
    a.q = a.k = a.w = a.idx = a.p = FAKE
    n = ctypes.c_size_t(0)
    f = L.lib().sa_indexer_kl_grad_get_workspace_size
    assert f(ctypes.byref(a), ctypes.byref(n)) == L.SA_OK
    assert n.value >= 2 * 64 * 128 * 4                                # the fp32 dk accumulator
    for field, val, want in (("n_heads", 48, L.SA_ERR_UNSUPPORTED), ("d", 96, L.SA_ERR_UNSUPPORTED),
                             ("topk", 0, L.SA_ERR_PARAM), ("p", None, L.SA_ERR_NULLPTR), ("layout", 9, L.SA_ERR_PARAM)):
        b = L.SaIndexerArgs.from_buffer_copy(a)
        setattr(b, field, val)
        assert f(ctypes.byref(b), ctypes.byref(n)) == want, field
    g = L.SaIndexerGrads(loss=None, dq=FAKE, dk=FAKE, dw=None)
    assert L.lib().sa_indexer_kl_grad(ctypes.byref(a), ctypes.byref(g), FAKE, 1 << 30, None) == L.SA_ERR_NULLPTR
    g.dw = FAKE
    assert L.lib().sa_indexer_kl_grad(ctypes.byref(a), ctypes.byref(g), FAKE, 16, None) == L.SA_ERR_WORKSPACE


def test_paged_cache_validates_on_the_host():
    """A paged KV cache: BSND only, page geometry covering s_kv, no compressed KV, and no
    backward (SA_ERR_UNSUPPORTED); checked before any device work."""
    ok = dict(block_table=FAKE, page_size=64, max_pages=2, t_kv=1024)
    n = ctypes.c_size_t(0)
    f = L.lib().sa_fwd_get_workspace_size
    assert f(ctypes.byref(_args(**ok)), ctypes.byref(n)) == L.SA_OK
    assert f(ctypes.byref(_args(**dict(ok, page_size=0))), ctypes.byref(n)) == L.SA_ERR_PARAM
    assert f(ctypes.byref(_args(**dict(ok, max_pages=1))), ctypes.byref(n)) == L.SA_ERR_PARAM   # 64 < s_kv
    assert f(ctypes.byref(_args(**dict(ok, t_kv=0))), ctypes.byref(n)) == L.SA_ERR_PARAM
    tnd = dict(ok, layout_q=L.SA_LAYOUT_TND, layout_kv=L.SA_LAYOUT_TND, t_q=8, cu_seqlens_q=FAKE,
               cu_seqlens_kv=FAKE)
    assert f(ctypes.byref(_args(**tnd)), ctypes.byref(n)) == L.SA_ERR_UNSUPPORTED
    assert L.lib().sa_bwd_get_workspace_size(ctypes.byref(_args(**ok)), ctypes.byref(n)) == L.SA_ERR_UNSUPPORTED
    # the block kernels do not take a paged cache: the generic forward does
    assert _plan(_args(**ok))[0] == L.SA_KERNEL_FWD_GENERIC


def test_softmax_l1norm_validates_on_the_host():
    """sa_softmax_l1norm needs an output, its index list, and the forward's lse; all
    checked before any device work (no GPU here)."""
    f = L.lib().sa_softmax_l1norm
    assert f(ctypes.byref(_args()), FAKE, None, None, None) == L.SA_ERR_NULLPTR
    assert f(ctypes.byref(_args()), None, FAKE, None, None) == L.SA_ERR_NULLPTR          # no lse
    assert f(ctypes.byref(_args(topk=0, ori_idx=None)), FAKE, FAKE, None, None) == L.SA_ERR_PARAM  # no ori indices
    assert f(ctypes.byref(_args()), FAKE, None, FAKE, None) == L.SA_ERR_PARAM             # no cmp indices
    assert f(ctypes.byref(_args(n_heads_q=15)), FAKE, FAKE, None, None) == L.SA_ERR_PARAM
    assert f(ctypes.byref(_args(s_q=0, s_kv=0)), None, FAKE, None, None) == L.SA_OK       # empty query


def test_status_and_inspection_calls_validate_on_the_host():
    assert L.lib().sa_read_status(None, 256, None) == L.SA_ERR_NULLPTR
    assert L.lib().sa_read_status(FAKE, 0, None) == L.SA_ERR_WORKSPACE
    n = FAKE
    dbi = L.lib().sa_debug_block_index
    assert dbi(ctypes.byref(_args()), 7, None, 0, FAKE, 16, n, None) == L.SA_ERR_PARAM
    assert dbi(ctypes.byref(_args()), L.SA_INDEX_VIEW_QUERY_BLOCKS, None, 0, FAKE, -1, n, None) == L.SA_ERR_PARAM
    assert dbi(ctypes.byref(_args()), L.SA_INDEX_VIEW_QUERY_BLOCKS, None, 0, FAKE, 16, None, None) == \
        L.SA_ERR_NULLPTR
    # the key-stationary view needs a backward workspace, and a problem that runs key-stationary
    assert dbi(ctypes.byref(_args()), L.SA_INDEX_VIEW_KEY_LISTS, None, 0, FAKE, 16, n, None) == L.SA_ERR_WORKSPACE
    assert dbi(ctypes.byref(_args(sinks=FAKE)), L.SA_INDEX_VIEW_KEY_LISTS, FAKE, 1 << 30, FAKE, 16, n, None) == \
        L.SA_ERR_UNSUPPORTED
    assert dbi(ctypes.byref(_args(block_size=16)), L.SA_INDEX_VIEW_QUERY_BLOCKS, None, 0, FAKE, 16, n, None) == \
        L.SA_ERR_UNSUPPORTED
