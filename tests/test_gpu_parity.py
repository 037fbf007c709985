"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
seeded inputs.  Small workloads compare every output element; the five
full-size workloads compare sampled units and tail KV rows in the launch
configuration the benchmark times."""

import numpy as np
import pytest
import torch

from gen import get_workload, make_inputs, scaled
from gpu_harness import run_full_comparison, run_sampled

pytestmark = pytest.mark.gpu


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for -m gpu tests")


SMALL = {
    "cfg1_full": (get_workload("cfg1"), {}),
    "cfg2_small": (scaled("cfg2", S=700, Hq=32, Hkv=2, seed=21), {}),
    "cfg2_future_len": (scaled("cfg2", "future", S=448, Hq=16, Hkv=1, seed=22),
                        dict(allow_future=True, ori_len_range=(0, 16))),
    "cfg3_small": (scaled("cfg3", S=700, Hq=32, topk=256, seed=23), {}),
    "cfg4_small": (scaled("cfg4", seqlens=(100, 300, 37), Hq=16, cmp_topk=64,
                          cmp_len_range=(16, 64), seed=24), {}),
    "cfg4_cmp_any_band": (scaled("cfg4", "any", seqlens=(130, 71), Hq=16, cmp_topk=32,
                                 cmp_len_range=(8, 32), win_left=40, win_right=5, seed=25),
                          dict(cmp_any=True)),
    "cfg5_small": (scaled("cfg5", S=2048, Hq=16, Hkv=4, seed=26), {}),
    "cfg5_empty_rows": (scaled("cfg5", "empty", S=512, Hq=8, Hkv=2, p_drop=0.6, seed=27), {}),
    "block_g24_128": (scaled("cfg2", "g24", S=320, Hq=48, Hkv=2, d_qk=128, d_v=128, topk=6,
                             seed=28), {}),
    "block_bs16_d64": (scaled("cfg1", "bs16", S=300, Hq=8, Hkv=2, block_size=16, topk=6,
                              seed=29), {}),
    "block_bs128_d64": (scaled("cfg1", "bs128", S=600, Hq=4, Hkv=1, block_size=128, topk=3,
                               seed=30), {}),
    "block_tnd": (scaled("cfg1", "tnd", layout="TND", seqlens=(200, 64, 333), Hq=8, Hkv=1,
                         seed=31), {}),
    "token_shared_128_nomask": (scaled("cfg3", "nomask", S=333, Hq=16, d_qk=128, d_v=128,
                                       topk=100, ori_mask="none", seed=32), {}),
    # token-level shared KV with 64 or 128 heads per KV head: the tcgen05 token kernel
    "token_h64_topk": (scaled("cfg3", "h64", S=400, Hq=64, topk=256, seed=35), {}),
    "token_h128_topk": (scaled("cfg3", "h128", S=300, Hq=128, topk=96, seed=36), {}),
    "swa_cmp_h64": (scaled("cfg4", "h64", seqlens=(100, 300, 37), Hq=64, cmp_topk=64,
                           cmp_len_range=(16, 64), seed=37), {}),
    # CFA: the window over the original KV plus every compressed row (no cmp indices), on the
    # generic kernels (16 heads) and the tcgen05 token kernels (64 heads)
    "cfa_h16": (scaled("cfg4", "cfa", seqlens=(100, 300, 37), Hq=16, cmp_topk=0, cmp_all=True, cmp_ratio=8,
                       seed=39), {}),
    "cfa_h64": (scaled("cfg4", "cfa64", seqlens=(200, 77), Hq=64, cmp_topk=0, cmp_all=True, cmp_ratio=8,
                       seed=40), {}),
    # sequsedQ / sequsedOriKv / sequsedCmpKv: padded sequences of which only the first
    # `used` tokens take part (generic kernels for blocks; tcgen05 token kernels at 64 heads)
    "block_used": (scaled("cfg1", "used", B=2, S=256, Hq=8, Hkv=2, topk=3, used=(200, 97), seed=41), {}),
    "token_used_h64": (scaled("cfg3", "used", S=400, Hq=64, topk=128, used=(301,), seed=42), {}),
    "swa_cmp_used": (scaled("cfg4", "used", seqlens=(100, 300, 37), Hq=16, cmp_topk=64, cmp_len_range=(16, 64),
                            used=(80, 213, 37), seed=43), {}),
    # 128 heads per KV head (window + compressed rows + sinks)
    "swa_cmp_h128": (scaled("cfg4", "h128", seqlens=(100, 300, 37), Hq=128, cmp_topk=64,
                            cmp_len_range=(16, 64), seed=38), {}),
    # G = 1 and 2: key-stationary tiles of 128 and 64 tokens with rows gathered one by one
    "block_g1_d64": (scaled("cfg1", "g1", S=700, Hq=2, Hkv=2, topk=5, seed=33), {}),
    "block_g2_d128": (scaled("cfg5", "g2", S=1000, Hq=4, Hkv=2, d_qk=128, d_v=128, topk=7, zipf_s=1.2,
                             p_drop=0.2, seed=34), dict(ori_len_range=(0, 7))),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_workload_all_elements(name):
    _need_gpu()
    w, kw = SMALL[name]
    run_full_comparison(w, kw)


BLOCK_CASES = ["cfg1_full", "cfg2_small", "cfg2_future_len", "cfg5_small", "cfg5_empty_rows", "block_g24_128",
               "block_g1_d64", "block_g2_d128"]


@pytest.mark.parametrize("flag", ["dq_separate", "query_stationary"])
@pytest.mark.parametrize("name", BLOCK_CASES)
def test_block_level_backward_variants(name, flag):
    """The block-level workloads through the other backward kernels: dQ from a separate
    query-stationary pass, and the fused query-stationary kernel."""
    _need_gpu()
    from top_sparse_attention_attn_b200 import _lib as L
    w, kw = SMALL[name]
    flags = {"dq_separate": L.SA_FLAG_DQ_SEPARATE, "query_stationary": L.SA_FLAG_QUERY_STATIONARY_BWD}[flag]
    run_full_comparison(w, kw, flags=flags)


@pytest.mark.parametrize("name", BLOCK_CASES)
def test_block_level_forward_on_tcgen05(name):
    """The block-level workloads through the tcgen05 forward (SA_FLAG_FWD_BLOCK_TC)."""
    _need_gpu()
    from top_sparse_attention_attn_b200 import _lib as L
    w, kw = SMALL[name]
    run_full_comparison(w, kw, flags=L.SA_FLAG_FWD_BLOCK_TC)


TOKEN_H128 = {
    **{k: SMALL[k] for k in ("token_h128_topk", "swa_cmp_h128")},
    # a 2048-token sequence with top-2048: every sub-tile pattern of the paired gathers
    "token_h128_s2048": (scaled("cfg3", "s2048", S=2048, Hq=128, seed=44), {}),
}


@pytest.mark.parametrize("name", list(TOKEN_H128))
def test_token_forward_pair_equals_unpaired(name):
    """128 heads per kv-head: the cluster-paired token forward (each CTA of a token
    gathers every other sub-tile and copies it to the other) gives bit-identical O
    and lse to the unpaired kernel (SA_FLAG_TOKEN_FWD_UNPAIRED), which the oracle
    comparison then checks element by element."""
    _need_gpu()
    from top_sparse_attention_attn_b200 import _lib as L
    from gpu_harness import device_problem
    w, kw = TOKEN_H128[name]
    inputs = make_inputs(w, **kw)
    res = []
    for flags in (0, L.SA_FLAG_TOKEN_FWD_UNPAIRED):
        sa, _ = device_problem(w, inputs, flags)
        assert sa.plan()[0] == L.SA_KERNEL_FWD_TOKEN_TC
        ws = sa.fwd_workspace()
        o, lse = sa.forward(ws=ws)
        torch.cuda.synchronize()
        assert sa.read_status(ws) == 0
        res.append((o.view(torch.int16).cpu().numpy(), lse.cpu().numpy()))
    np.testing.assert_array_equal(res[0][0], res[1][0])
    np.testing.assert_array_equal(res[0][1], res[1][1])
    if name != "token_h128_s2048":
        run_full_comparison(w, kw, flags=L.SA_FLAG_TOKEN_FWD_UNPAIRED)


@pytest.mark.parametrize("cfg", ["cfg2", "cfg1", "cfg5", "cfg4", "cfg3"])
def test_full_size_sampled(cfg):
    _need_gpu()
    w = get_workload(cfg)
    tail = 16 if cfg == "cfg3" else 64
    run_sampled(w, n_units=16 if cfg == "cfg3" else 24, tail_rows=tail)


@pytest.mark.parametrize("name", ["cfg2_small", "cfg4_small"])
def test_calls_capture_in_a_cuda_graph(name):
    """sa_fwd / sa_bwd enqueue only kernels and memsets on the caller's stream, so a
    CUDA graph of them replays to the same results as the eager calls."""
    _need_gpu()
    from gpu_harness import check_close, device_problem, grads_to_host, widen
    from gen.torch_io import bf16_bits
    w, kw = SMALL[name]
    sa, t = device_problem(w, make_inputs(w, **kw))
    o, lse = sa.alloc_fwd()
    grads = sa.alloc_bwd()
    ws_f, ws_b = sa.fwd_workspace(), sa.bwd_workspace()
    sa.forward(o, lse, ws_f)
    sa.backward(o, lse, t["do"], grads, ws_b)
    torch.cuda.synchronize()
    ref_o, ref_lse, ref_g = bf16_bits(o), lse.cpu().numpy(), grads_to_host(grads)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g1, g2 = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g1):
            sa.forward(o, lse, ws_f)
        with torch.cuda.graph(g2):
            sa.backward(o, lse, t["do"], grads, ws_b)
    torch.cuda.current_stream().wait_stream(side)
    o.fill_(float("nan"))
    for v in grads.values():
        v.fill_(float("nan"))
    for _ in range(2):
        g1.replay()
        g2.replay()
    torch.cuda.synchronize()
    check_close("graph:O", widen(bf16_bits(o)), widen(ref_o))
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=1e-5)
    got = grads_to_host(grads)
    for key in ref_g:
        if key == "dsinks":
            check_close(f"graph:{key}", got[key], ref_g[key])
        else:
            check_close(f"graph:{key}", widen(got[key]), widen(ref_g[key]))


def _with_duplicates(inputs, key, every=3):
    """A copy of the inputs in which, for every ``every``-th (token, kv-head) list, slot 1
    repeats slot 0's index when slot 0 is in use (a selection that names a row or block
    twice)."""
    out = dict(inputs)
    idx = np.array(inputs[key], copy=True)
    flat = idx.reshape(-1, idx.shape[-1])
    rows = np.arange(0, flat.shape[0], every)
    take = rows[flat[rows, 0] >= 0]
    flat[take, 1] = flat[take, 0]
    out[key] = idx
    return out, len(take)


DUP_CASES = {
    "token_h64_dup": ("token_h64_topk", "ori_idx"),      # tcgen05 token kernels
    "block_cfg2_dup": ("cfg2_small", "ori_idx"),         # TMA-fed block forward, key-stationary backward
    "block_bs16_dup": ("block_bs16_d64", "ori_idx"),     # generic kernels
    "swa_cmp_dup": ("swa_cmp_h64", "cmp_idx"),           # token kernels, repeated compressed rows
}


@pytest.mark.parametrize("name", list(DUP_CASES))
def test_duplicate_indices_count_twice(name):
    """A row or block named twice in one selection list contributes twice, as the oracle's
    slot-by-slot gather counts it (duplicate indices are taken with multiplicity)."""
    _need_gpu()
    base, key = DUP_CASES[name]
    w, kw = SMALL[base]
    inputs, n = _with_duplicates(make_inputs(w, **kw), key)
    assert n > 0
    run_full_comparison(w, inputs=inputs)
