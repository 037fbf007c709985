"""ctypes binding of libsparse_attn.so (include/sparse_attn.h).

Argument marshalling only: every entry point here converts Python values into
the C structs and calls the library; all computation happens in the CUDA
kernels behind the C ABI.  Loading fails loudly when the library is missing.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsparse_attn.so")

SA_OK = 0
SA_ERR_NULLPTR = 1
SA_ERR_PARAM = 2
SA_ERR_UNSUPPORTED = 3
SA_ERR_WORKSPACE = 4
SA_ERR_INDEX = 5
SA_ERR_TIMEOUT = 6
SA_ERR_CUDA = 7

SA_LAYOUT_BSND = 0
SA_LAYOUT_TND = 1
SA_MASK_NONE = 0
SA_MASK_CAUSAL = 1
SA_MASK_BAND = 2
SA_DTYPE_BF16 = 0
SA_DTYPE_FP16 = 1
SA_FLAG_CHECK = 1
SA_FLAG_QUERY_STATIONARY_BWD = 2
SA_FLAG_DQ_SEPARATE = 4
SA_FLAG_FWD_BLOCK_TC = 8
SA_FLAG_TOKEN_FWD_UNPAIRED = 16

# sa_kernel (sa_plan)
SA_KERNEL_FWD_BLOCK = 1
SA_KERNEL_FWD_TOKEN_TC = 2
SA_KERNEL_FWD_GENERIC = 3
SA_KERNEL_BWD_KEY_STATIONARY = 4
SA_KERNEL_BWD_KEY_STATIONARY_DQ_PASS = 5
SA_KERNEL_BWD_TOKEN_TC = 6
SA_KERNEL_BWD_GENERIC = 7
SA_KERNEL_FWD_BLOCK_TC = 8
SA_INDEX_VIEW_QUERY_BLOCKS = 0
SA_INDEX_VIEW_KEY_LISTS = 1

# status word bits (the first 4 bytes of every workspace)
SA_STATUS_INDEX = 1
SA_STATUS_TIMEOUT = 2
SA_STATUS_SMEM_ALIGN = 4

MASKS = {"none": SA_MASK_NONE, "causal": SA_MASK_CAUSAL, "band": SA_MASK_BAND}
LAYOUTS = {"BSND": SA_LAYOUT_BSND, "TND": SA_LAYOUT_TND}

_vp = ctypes.c_void_p
_ip = ctypes.POINTER(ctypes.c_int32)
_fp = ctypes.POINTER(ctypes.c_float)


class SaArgs(ctypes.Structure):
    _fields_ = [
        ("layout_q", ctypes.c_int32), ("layout_kv", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("s_q", ctypes.c_int32), ("s_kv", ctypes.c_int32),
        ("t_q", ctypes.c_int32), ("t_kv", ctypes.c_int32), ("t_cmp", ctypes.c_int32),
        ("n_heads_q", ctypes.c_int32), ("n_heads_kv", ctypes.c_int32),
        ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32), ("kv_shared", ctypes.c_int32),
        ("block_size", ctypes.c_int32), ("topk", ctypes.c_int32), ("cmp_topk", ctypes.c_int32),
        ("cmp_ratio", ctypes.c_int32), ("ori_mask_mode", ctypes.c_int32),
        ("cmp_mask_mode", ctypes.c_int32), ("ori_win_left", ctypes.c_int64),
        ("ori_win_right", ctypes.c_int64), ("scale", ctypes.c_float), ("flags", ctypes.c_uint32),
        ("q", _vp), ("k", _vp), ("v", _vp), ("kv", _vp), ("cmp_kv", _vp),
        ("ori_idx", _vp), ("cmp_idx", _vp),
        ("cu_seqlens_q", _vp), ("cu_seqlens_kv", _vp), ("cu_seqlens_cmp", _vp),
        ("ori_topk_len", _vp), ("cmp_topk_len", _vp), ("cmp_residual", _vp), ("sinks", _vp),
        ("seqused_q", _vp), ("seqused_kv", _vp), ("seqused_cmp", _vp),
        ("block_table", _vp), ("page_size", ctypes.c_int32), ("max_pages", ctypes.c_int32),
    ]


class SaIndexerArgs(ctypes.Structure):
    _fields_ = [
        ("layout", ctypes.c_int32), ("batch", ctypes.c_int32), ("s_q", ctypes.c_int32), ("s_kv", ctypes.c_int32),
        ("t_q", ctypes.c_int32), ("t_kv", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("d", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("q", _vp), ("k", _vp), ("w", _vp), ("idx", _vp), ("topk_len", _vp), ("p", _vp),
        ("cu_seqlens_q", _vp), ("cu_seqlens_kv", _vp),
    ]


class SaIndexerGrads(ctypes.Structure):
    _fields_ = [("loss", _vp), ("dq", _vp), ("dk", _vp), ("dw", _vp)]


class SaFwdOut(ctypes.Structure):
    _fields_ = [("o", _vp), ("lse", _vp)]


class SaBwdIo(ctypes.Structure):
    _fields_ = [("o", _vp), ("d_o", _vp), ("lse", _vp), ("dq", _vp), ("dk", _vp), ("dv", _vp),
                ("dkv", _vp), ("dcmp_kv", _vp), ("dsinks", _vp)]


class SaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


_lib = None

# every symbol include/sparse_attn.h declares
EXPORTS = ["sa_fwd_get_workspace_size", "sa_fwd", "sa_bwd_get_workspace_size", "sa_bwd",
           "sa_softmax_grad_preprocess", "sa_debug_resolve", "sa_status_string", "sa_abi_version",
           "sa_set_timing_events", "sa_kernel_launch_count", "sa_bwd_no_alloc",
           "sa_bwd_no_alloc_max_workspace", "sa_selftest_mma", "sa_selftest_wait_timeout",
           "sa_selftest_mma2", "sa_plan", "sa_read_status", "sa_bwd_no_alloc_read_status",
           "sa_debug_block_index", "sa_selftest_gather4", "sa_softmax_l1norm",
           "sa_indexer_kl_grad_get_workspace_size", "sa_indexer_kl_grad"]


def lib() -> ctypes.CDLL:
    """Load libsparse_attn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m top_sparse_attention_attn_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        L.sa_fwd_get_workspace_size.argtypes = [P(SaArgs), P(ctypes.c_size_t)]
        L.sa_fwd.argtypes = [P(SaArgs), P(SaFwdOut), _vp, ctypes.c_size_t, _vp]
        L.sa_bwd_get_workspace_size.argtypes = [P(SaArgs), P(ctypes.c_size_t)]
        L.sa_bwd.argtypes = [P(SaArgs), P(SaBwdIo), _vp, ctypes.c_size_t, _vp]
        L.sa_softmax_grad_preprocess.argtypes = [P(SaArgs), _vp, _vp, _vp, _vp]
        L.sa_softmax_l1norm.argtypes = [P(SaArgs), _vp, _vp, _vp, _vp]
        L.sa_indexer_kl_grad_get_workspace_size.argtypes = [P(SaIndexerArgs), P(ctypes.c_size_t)]
        L.sa_indexer_kl_grad.argtypes = [P(SaIndexerArgs), P(SaIndexerGrads), _vp, ctypes.c_size_t, _vp]
        L.sa_debug_resolve.argtypes = [P(SaArgs), _vp, _vp, ctypes.c_int32, _vp]
        L.sa_status_string.argtypes = [ctypes.c_int32]
        L.sa_status_string.restype = ctypes.c_char_p
        L.sa_abi_version.argtypes = []
        L.sa_set_timing_events.argtypes = [_vp, _vp, ctypes.c_int32]
        L.sa_set_timing_events.restype = None
        L.sa_kernel_launch_count.argtypes = []
        L.sa_kernel_launch_count.restype = ctypes.c_int64
        L.sa_bwd_no_alloc.argtypes = [P(SaArgs), P(SaBwdIo), _vp]
        L.sa_bwd_no_alloc_max_workspace.argtypes = []
        L.sa_bwd_no_alloc_max_workspace.restype = ctypes.c_size_t
        L.sa_selftest_mma.argtypes = [ctypes.c_int32] * 7 + [_vp, _vp, _vp, _vp, _vp]
        L.sa_selftest_wait_timeout.argtypes = [_vp, _vp, _vp]
        L.sa_selftest_mma2.argtypes = [ctypes.c_int32] * 8 + [_vp, _vp, _vp, _vp, _vp]
        L.sa_plan.argtypes = [P(SaArgs), _ip, _ip]
        L.sa_selftest_gather4.argtypes = [_vp, ctypes.c_int32, ctypes.c_int32, _vp, ctypes.c_int32, _vp, _vp, _vp]
        L.sa_read_status.argtypes = [_vp, ctypes.c_size_t, _vp]
        L.sa_bwd_no_alloc_read_status.argtypes = [_vp]
        L.sa_debug_block_index.argtypes = [P(SaArgs), ctypes.c_int32, _vp, ctypes.c_size_t, _vp, ctypes.c_int64,
                                           _vp, _vp]
        for name in EXPORTS:
            if name not in ("sa_status_string", "sa_set_timing_events", "sa_kernel_launch_count",
                            "sa_bwd_no_alloc_max_workspace"):
                getattr(L, name).restype = ctypes.c_int32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().sa_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != SA_OK:
        raise SaError(status, where)


# ---- the entry points, same names as the C ABI -------------------------------

def sa_fwd_get_workspace_size(args: SaArgs) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().sa_fwd_get_workspace_size(ctypes.byref(args), ctypes.byref(n)), "sa_fwd_get_workspace_size")
    return n.value


def sa_fwd(args: SaArgs, out: SaFwdOut, ws: int, ws_bytes: int, stream: int = 0) -> None:
    _check(lib().sa_fwd(ctypes.byref(args), ctypes.byref(out), ws, ws_bytes, stream), "sa_fwd")


def sa_bwd_get_workspace_size(args: SaArgs) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().sa_bwd_get_workspace_size(ctypes.byref(args), ctypes.byref(n)), "sa_bwd_get_workspace_size")
    return n.value


def sa_bwd(args: SaArgs, io: SaBwdIo, ws: int, ws_bytes: int, stream: int = 0) -> None:
    _check(lib().sa_bwd(ctypes.byref(args), ctypes.byref(io), ws, ws_bytes, stream), "sa_bwd")


def sa_bwd_no_alloc(args: SaArgs, io: SaBwdIo, stream: int = 0) -> None:
    """Backward on the library's fixed scratch array (no workspace, no allocation)."""
    _check(lib().sa_bwd_no_alloc(ctypes.byref(args), ctypes.byref(io), stream), "sa_bwd_no_alloc")


def sa_bwd_no_alloc_max_workspace() -> int:
    return int(lib().sa_bwd_no_alloc_max_workspace())


def sa_selftest_mma(M: int, N: int, K: int, a_mn: int, b_mn: int, box_rows: int, A: int, B: int,
                    D: int, status: int, stream: int = 0, d_lane: int = 0) -> None:
    _check(lib().sa_selftest_mma(M, N, K, a_mn, b_mn, box_rows, d_lane, A, B, D, status, stream),
           "sa_selftest_mma")


def sa_selftest_mma2(M: int, N: int, K: int, a_mn: int, b_mn: int, a_sw: int, b_sw: int, A: int, B: int,
                     D: int, status: int, stream: int = 0, d_lane: int = 0) -> None:
    _check(lib().sa_selftest_mma2(M, N, K, a_mn, b_mn, a_sw, b_sw, d_lane, A, B, D, status, stream),
           "sa_selftest_mma2")


def sa_selftest_gather4(src: int, rows: int, cols: int, row_idx: int, n: int, out: int, status: int,
                        stream: int = 0) -> None:
    _check(lib().sa_selftest_gather4(src, rows, cols, row_idx, n, out, status, stream), "sa_selftest_gather4")


def sa_selftest_wait_timeout(status: int, waited: int, stream: int = 0) -> None:
    _check(lib().sa_selftest_wait_timeout(status, waited, stream), "sa_selftest_wait_timeout")


def sa_softmax_grad_preprocess(args: SaArgs, o: int, d_o: int, delta: int, stream: int = 0) -> None:
    _check(lib().sa_softmax_grad_preprocess(ctypes.byref(args), o, d_o, delta, stream),
           "sa_softmax_grad_preprocess")


def sa_indexer_kl_grad_get_workspace_size(args: SaIndexerArgs) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().sa_indexer_kl_grad_get_workspace_size(ctypes.byref(args), ctypes.byref(n)),
           "sa_indexer_kl_grad_get_workspace_size")
    return n.value


def sa_indexer_kl_grad(args: SaIndexerArgs, grads: SaIndexerGrads, ws: int, ws_bytes: int, stream: int = 0) -> None:
    _check(lib().sa_indexer_kl_grad(ctypes.byref(args), ctypes.byref(grads), ws, ws_bytes, stream),
           "sa_indexer_kl_grad")


def sa_softmax_l1norm(args: SaArgs, lse: int, ori_out, cmp_out, stream: int = 0) -> None:
    _check(lib().sa_softmax_l1norm(ctypes.byref(args), lse, ori_out, cmp_out, stream), "sa_softmax_l1norm")


def sa_debug_resolve(args: SaArgs, rows: int, counts: int, max_rows: int, stream: int = 0) -> None:
    _check(lib().sa_debug_resolve(ctypes.byref(args), rows, counts, max_rows, stream), "sa_debug_resolve")


def sa_plan(args: SaArgs) -> tuple:
    """(forward kernel, backward kernel) as SA_KERNEL_* values."""
    f, b = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib().sa_plan(ctypes.byref(args), ctypes.byref(f), ctypes.byref(b)), "sa_plan")
    return f.value, b.value


def sa_read_status(ws: int, ws_bytes: int, stream: int = 0) -> int:
    """The workspace status word mapped to an sa_status (synchronises the stream; never raises)."""
    return int(lib().sa_read_status(ws, ws_bytes, stream))


def sa_bwd_no_alloc_read_status(stream: int = 0) -> int:
    return int(lib().sa_bwd_no_alloc_read_status(stream))


def sa_debug_block_index(args: SaArgs, view: int, ws: int, ws_bytes: int, records: int, max_records: int,
                         n_records: int, stream: int = 0) -> None:
    _check(lib().sa_debug_block_index(ctypes.byref(args), view, ws, ws_bytes, records, max_records, n_records,
                                      stream), "sa_debug_block_index")


def sa_abi_version() -> int:
    return int(lib().sa_abi_version())


TIME_FWD, TIME_BWD_KV, TIME_BWD_DQ = 0, 1, 2


def sa_set_timing_events(ev_begin: int | None, ev_end: int | None, which: int = TIME_BWD_KV) -> None:
    lib().sa_set_timing_events(ev_begin, ev_end, which)


def sa_kernel_launch_count() -> int:
    return int(lib().sa_kernel_launch_count())
