"""Bit-exact checks of the block-level index sets the kernels actually use.

The visible set of every (query token, kv-head) unit is fixed by the Gather
through topkIndices (aclnnSparseFlashAttentionGrad, "Formula") together with
the topk lengths and the masks (SparseFlashMlaGrad, "Parameter Description").
sa_debug_block_index returns that set as the block kernels build it:
  - the query-stationary view runs the block kernels' own slot rule and
    in-block row range, unit by unit;
  - the key-stationary view builds the backward's inverse index (the bucketed
    one-launch index for small problems, count / scan / fill otherwise) and
    walks every work item as the backward kernel does.
Both must equal the oracle's visible rows exactly.  The status word and the
SA_FLAG_CHECK path are checked here too, with indices past their sequence
(which the kernels never read: they select nothing).
"""

import numpy as np
import pytest
import torch

import oracle
from gen import get_workload, make_inputs, scaled
from gpu_harness import device_problem
from top_sparse_attention_attn_b200 import _lib as L

pytestmark = pytest.mark.gpu

CASES = {
    "cfg1_full": (get_workload("cfg1"), {}),                                    # bucketed index
    "cfg2_small": (scaled("cfg2", S=700, Hq=32, Hkv=2, seed=21), {}),            # count / scan / fill
    "cfg2_future_len": (scaled("cfg2", "future", S=448, Hq=16, Hkv=1, seed=22),
                        dict(allow_future=True, ori_len_range=(0, 16))),
    "cfg5_empty_rows": (scaled("cfg5", "empty", S=512, Hq=8, Hkv=2, p_drop=0.6, seed=27), {}),
    "block_band": (scaled("cfg1", "band", S=640, Hq=8, Hkv=2, topk=6, ori_mask="band", win_left=100,
                          win_right=40, seed=51), dict(allow_future=True)),
    "block_nomask_future": (scaled("cfg1", "nomask", S=500, Hq=4, Hkv=1, topk=5, ori_mask="none", seed=52),
                            dict(allow_future=True, ori_len_range=(0, 5))),
    "block_g2_len": (scaled("cfg5", "g2", S=1000, Hq=4, Hkv=2, d_qk=128, d_v=128, topk=7, zipf_s=1.2,
                            p_drop=0.2, seed=34), dict(ori_len_range=(0, 7))),
    # S = 8192: count / scan / fill over two token windows (dQ rows of a window kept in L2)
    "cfg2_s8192_windows": (scaled("cfg2", "win", B=1, S=8192, Hq=16, Hkv=1, seed=53), {}),
}


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for -m gpu tests")


def _rows_by_unit(rec: np.ndarray, n_units: int) -> list:
    assert rec.ndim == 2 and rec.shape[1] == 4
    unit, x, lo, hi = rec[:, 0].astype(np.int64), rec[:, 1].astype(np.int64), rec[:, 2], rec[:, 3]
    assert np.all((unit >= 0) & (unit < n_units)), "record for a unit out of range"
    assert np.all((lo >= 0) & (lo <= hi) & (hi < 64)), "empty or out-of-block row range"
    out = [[] for _ in range(n_units)]
    for u, xx, a, b in zip(unit.tolist(), x.tolist(), lo.tolist(), hi.tolist()):
        out[u].append(np.arange(64 * xx + a, 64 * xx + b + 1, dtype=np.int64))
    return [np.sort(np.concatenate(r)) if r else np.zeros(0, dtype=np.int64) for r in out]


def _check_view(name, sa, p, w, view):
    rec = sa.block_index(view).cpu().numpy()
    n_units = w.T * w.Hkv
    got = _rows_by_unit(rec, n_units)
    for u in range(n_units):
        tq, g = divmod(u, w.Hkv)
        ref = np.sort(oracle.visible_rows(p, tq, g)[0].astype(np.int64))
        if not np.array_equal(got[u], ref):
            raise AssertionError(f"{name} view {view}: unit {(tq, g)} has {len(got[u])} visible rows, "
                                 f"oracle {len(ref)}; first difference in "
                                 f"{np.setxor1d(got[u], ref)[:8].tolist()}")
    return len(rec)


@pytest.mark.parametrize("name", list(CASES))
def test_block_index_sets_are_exact(name):
    _need_gpu()
    w, kw = CASES[name]
    inputs = make_inputs(w, **kw)
    p = oracle.Problem.from_inputs(w, inputs)
    sa, _ = device_problem(w, inputs)
    fwd_k, bwd_k = sa.plan()
    checked = 0
    if fwd_k == L.SA_KERNEL_FWD_BLOCK:
        _check_view(name, sa, p, w, L.SA_INDEX_VIEW_QUERY_BLOCKS)
        checked += 1
    if bwd_k in (L.SA_KERNEL_BWD_KEY_STATIONARY, L.SA_KERNEL_BWD_KEY_STATIONARY_DQ_PASS):
        _check_view(name, sa, p, w, L.SA_INDEX_VIEW_KEY_LISTS)
        checked += 1
    assert checked == 2, f"{name}: plan {(fwd_k, bwd_k)} does not run both block kernels"


def _bad_index_inputs(w, kw, where):
    inputs = make_inputs(w, **kw)
    T = w.T
    if where == "ori":
        idx = inputs["ori_idx"].reshape(T, w.Hkv, -1)
        nblk = -(-max(w.seq_lengths) // max(w.block_size, 1))
        idx[T // 2, 0, 0] = nblk + 3          # past the end of the sequence
        idx[T - 1, w.Hkv - 1, -1] = nblk      # the first block past the end
    else:
        cidx = inputs["cmp_idx"].reshape(T, w.Hkv, -1)
        cidx[T // 2, 0, 0] = max(w.seq_lengths) // w.cmp_ratio + 5
    return inputs


@pytest.mark.parametrize("name,where", [("cfg1_full", "ori"), ("cfg2_small", "ori"), ("cfg4_small", "cmp")])
def test_indices_past_the_sequence_are_reported(name, where):
    """SA_FLAG_CHECK returns SA_ERR_INDEX before computing; without it the call runs
    (such indices select nothing) and sa_read_status reports SA_ERR_INDEX."""
    _need_gpu()
    if name == "cfg4_small":
        w, kw = scaled("cfg4", seqlens=(100, 300, 37), Hq=16, cmp_topk=64, cmp_len_range=(64, 64),
                       seed=24), {}
    else:
        w, kw = CASES[name]
    inputs = _bad_index_inputs(w, kw, where)
    sa, t = device_problem(w, inputs, flags=L.SA_FLAG_CHECK)
    with pytest.raises(L.SaError) as e:
        sa.forward()
    assert e.value.status == L.SA_ERR_INDEX
    sa.flags = 0
    ws_f = sa.fwd_workspace()
    o, lse = sa.forward(ws=ws_f)
    assert sa.read_status(ws_f) == L.SA_ERR_INDEX
    ws_b = sa.bwd_workspace()
    grads = sa.backward(o, lse, t["do"], ws=ws_b)
    assert sa.read_status(ws_b) == L.SA_ERR_INDEX
    for v in grads.values():
        assert torch.isfinite(v.float()).all()
    # a clean problem leaves the word clear
    clean, t2 = device_problem(w, make_inputs(w, **kw))
    ws_f2, ws_b2 = clean.fwd_workspace(), clean.bwd_workspace()
    o2, lse2 = clean.forward(ws=ws_f2)
    clean.backward(o2, lse2, t2["do"], ws=ws_b2)
    assert clean.read_status(ws_f2) == L.SA_OK
    assert clean.read_status(ws_b2) == L.SA_OK
