"""The tensor-core building blocks (TMA tile loads into 128-byte swizzled
shared memory, matrix descriptors for K-major and MN-major operands,
tcgen05.mma, TMEM accumulators of height 64 and 128) against a plain fp32
matmul of the same bf16 operands."""

import pytest
import torch

from top_sparse_attention_attn_b200 import _lib as L

pytestmark = pytest.mark.gpu

CASES = [
    # M, N, K, a_mn, b_mn, box_rows[, d_lane]
    (128, 64, 64, 0, 0, 64), (128, 64, 192, 0, 0, 16), (128, 256, 128, 0, 0, 8),
    (128, 64, 128, 1, 1, 64), (128, 64, 128, 1, 1, 16), (64, 64, 128, 1, 1, 32),
    (128, 192, 64, 0, 1, 64), (128, 128, 256, 1, 0, 16), (64, 128, 64, 0, 0, 8),
    (64, 192, 128, 1, 1, 64), (128, 192, 128, 1, 0, 8),
    (64, 64, 128, 1, 1, 64, 16), (64, 128, 64, 0, 0, 16, 16),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_tcgen05_mma_matches_matmul(case):
    M, N, K, a_mn, b_mn, box = case[:6]
    d_lane = case[6] if len(case) > 6 else 0
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for -m gpu tests")
    g = torch.Generator(device="cuda").manual_seed(M * 1000 + N * 10 + K + a_mn + 2 * b_mn)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, device="cuda", generator=g).to(torch.bfloat16)
    a_store = A.t().contiguous() if a_mn else A.contiguous()          # [K][M] or [M][K]
    b_store = B.contiguous() if b_mn else B.t().contiguous()          # [K][N] or [N][K]
    D = torch.full((M, N), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.sa_selftest_mma(M, N, K, a_mn, b_mn, box, a_store.data_ptr(), b_store.data_ptr(), D.data_ptr(),
                      status.data_ptr(), torch.cuda.current_stream().cuda_stream, d_lane=d_lane)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = A.float() @ B.float()
    err = (D - ref).abs().max().item()
    assert err <= 1e-3 * ref.abs().max().item(), f"max err {err}"


@pytest.mark.gpu
def test_bounded_wait_gives_up_and_reports():
    """A wait on an mbarrier that nothing arrives on gives up after its poll limit: the
    kernel raises the status word's timeout bit and ends normally, and the context keeps
    working (a tensor-core self-check right after still computes correctly)."""
    import time
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    L.sa_selftest_wait_timeout(status.data_ptr(), waited.data_ptr())
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert int(waited.item()) == 0, "the wait completed although nothing arrived"
    assert int(status.item()) & 2, "the timeout bit was not raised"
    assert elapsed < 20.0, f"the bounded wait took {elapsed:.1f} s"
    print(f"bounded wait gave up after {elapsed:.2f} s")
    # the word reads back through the ABI as SA_ERR_TIMEOUT (a status word of its own:
    # sa_read_status reads the first 4 bytes of any workspace)
    assert L.sa_read_status(status.data_ptr(), 4, torch.cuda.current_stream().cuda_stream) == L.SA_ERR_TIMEOUT
    status.zero_()
    assert L.sa_read_status(status.data_ptr(), 4, torch.cuda.current_stream().cuda_stream) == L.SA_OK
    test_tcgen05_mma_matches_matmul((128, 64, 64, 0, 0, 64))


CASES2 = [
    # M, N, K, a_mn, b_mn, a_sw, b_sw[, d_lane]: the token-level kernel's operand shapes
    (64, 32, 128, 0, 0, 128, 128), (64, 32, 128, 0, 0, 128, 128, 16),   # S / dP: 32-row K-major B
    (64, 256, 32, 0, 1, 64, 128), (64, 64, 32, 0, 1, 64, 128),          # dQ: 64-byte-swizzle A, K = 32
    (64, 256, 32, 0, 1, 64, 128, 16),                                   # dQ upper half at lane offset 16
    (128, 32, 64, 1, 1, 128, 64), (64, 32, 64, 1, 1, 128, 64),          # dKV: MN-major B of one 32-wide atom
    (128, 64, 128, 0, 0, 128, 128), (128, 128, 64, 1, 1, 128, 128),     # the TMA-loaded cases, loaded in software
    # the block forward's transposed operands: S^T = K Q^T (M = 64 keys, N = 16 heads, at
    # lane offsets 0 and 16) and O^T += V^T P^T (M = d_v as an MN-major A, P^T K-major)
    (64, 16, 192, 0, 0, 128, 128), (64, 16, 128, 0, 0, 128, 128, 16), (64, 16, 64, 0, 0, 128, 128),
    (128, 16, 64, 1, 0, 128, 128), (64, 16, 64, 1, 0, 128, 128),
]


@pytest.mark.parametrize("case", CASES2, ids=[str(c) for c in CASES2])
def test_software_layouts_match_matmul(case):
    M, N, K, a_mn, b_mn, a_sw, b_sw = case[:7]
    d_lane = case[7] if len(case) > 7 else 0
    g = torch.Generator(device="cuda").manual_seed(M * 1000 + N * 10 + K + a_sw + b_sw)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, device="cuda", generator=g).to(torch.bfloat16)
    a_store = A.t().contiguous() if a_mn else A.contiguous()
    b_store = B.contiguous() if b_mn else B.t().contiguous()
    D = torch.full((M, N), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.sa_selftest_mma2(M, N, K, a_mn, b_mn, a_sw, b_sw, a_store.data_ptr(), b_store.data_ptr(), D.data_ptr(),
                       status.data_ptr(), torch.cuda.current_stream().cuda_stream, d_lane=d_lane)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = A.float() @ B.float()
    err = (D - ref).abs().max().item()
    assert err <= 1e-3 * ref.abs().max().item(), f"max err {err}"


@pytest.mark.parametrize("cols,n", [(576, 32), (128, 8), (64, 4)])
def test_tma_row_gather_matches_index_select(cols, n):
    """tile::gather4 copies land each named row in the 128-byte-swizzled slab layout the
    tensor-core operands use (rows repeated and row 0 included)."""
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for -m gpu tests")
    rows = 1000
    g = torch.Generator(device="cuda").manual_seed(cols + n)
    src = torch.randn(rows, cols, device="cuda", generator=g).to(torch.bfloat16)
    idx = torch.randint(0, rows, (n,), device="cuda", generator=g, dtype=torch.int32)
    idx[0] = 0
    idx[-1] = rows - 1
    if n >= 8:
        idx[3] = idx[2]
    out = torch.full((n, cols), float("nan"), device="cuda").to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.sa_selftest_gather4(src.data_ptr(), rows, cols, idx.data_ptr(), n, out.data_ptr(), status.data_ptr(),
                          torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(out.view(torch.int16), src[idx.long()].view(torch.int16))
