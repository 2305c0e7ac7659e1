"""tcgen05 GEMM unit test through the C ABI (gdit_test_gemm): C = A B^T + bias
against float64 products of the same bf16 inputs."""

import numpy as np
import pytest

from tests.gpu_util import require_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K,bn,splits", [
    (128, 128, 64, 128, 1),        # one tile, one K block
    (200, 256, 192, 64, 1),        # ragged M, several N tiles, 3 K blocks
    (17, 1024, 1024, 64, 4),       # small-M weight streaming with split-K
    (300, 512, 2048, 256, 1),      # wide tiles, long K
    (1000, 96, 40, 32, 1),         # K below one block (zero-filled tail), narrow N
    (4352, 1024, 1024, 256, 1),    # persistent: more tiles than SMs
    (65, 4096, 512, 128, 3),       # split-K with a ragged row tile
])
@pytest.mark.parametrize("tma_out", [False, True])
def test_gemm_matches_float64(M, N, K, bn, splits, tma_out, monkeypatch):
    """tma_out: the epilogue stages 32-row boxes in shared memory and stores them by TMA."""
    require_gpu()
    if tma_out:
        if splits > 1 or bn < 64:
            pytest.skip("the TMA-store epilogue serves single-split tiles of width >= 64")
        monkeypatch.setenv("GDIT_TEST_TMA_OUT", "1")
    import torch
    from flow_matching_dit_b200 import test_gemm
    g = torch.Generator().manual_seed(M * 7 + N + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16)
    bias = torch.randn(N, generator=g)
    C = test_gemm(A.cuda(), B.cuda(), bias.cuda(), bn=bn, splits=splits).cpu().double().numpy()
    ref = A.double().numpy() @ B.double().numpy().T + bias.double().numpy()
    # f32 accumulation of exact bf16 products: error ~ sqrt(K) * 2^-24 * |terms|
    np.testing.assert_allclose(C, ref, rtol=1e-5, atol=2e-5 * np.sqrt(K))


@pytest.mark.parametrize("M,N,K,bn", [
    (256, 256, 64, 256),           # one pair tile, one K block
    (4352, 1024, 1024, 256),       # the DiT shape at B = 256 (17 row blocks of 256)
    (4352, 4096, 1024, 256),       # FF1: more pair tiles than clusters (persistent)
    (544, 3072, 1024, 256),        # ragged last row block (544 = 2 x 256 + 32)
    (300, 512, 2048, 128),         # narrow pair tiles, long K, ragged rows
    (130, 256, 40, 128),           # the odd CTA's rows mostly past the end; K below one block
])
def test_pair_gemm_matches_float64(M, N, K, bn, monkeypatch):
    """The CTA-pair kernel (cta_group::2 MMAs over two SMs, 256-row tiles,
    TMA-store epilogue) against float64 products of the same bf16 inputs."""
    require_gpu()
    monkeypatch.setenv("GDIT_TEST_TMA_OUT", "1")
    monkeypatch.setenv("GDIT_TEST_PAIR", "1")
    import torch
    from flow_matching_dit_b200 import test_gemm
    g = torch.Generator().manual_seed(M * 5 + N + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16)
    bias = torch.randn(N, generator=g)
    C = test_gemm(A.cuda(), B.cuda(), bias.cuda(), bn=bn, splits=1).cpu().double().numpy()
    ref = A.double().numpy() @ B.double().numpy().T + bias.double().numpy()
    np.testing.assert_allclose(C, ref, rtol=1e-5, atol=2e-5 * np.sqrt(K))


@pytest.mark.parametrize("M,N,K,plan", [
    (17, 1024, 1024, "2,1"),       # one sample's rows, one unit per item
    (136, 1024, 1024, "2,5"),      # eight samples: 32-row blocks, ragged last block (8 rows)
    (136, 4096, 1024, "3,6"),      # 258 items: CTAs take several items (pipeline across items)
    (34, 384, 128, "1,16"),        # K of half a chunk (boxes past K read zeros)
    (85, 96, 320, "5,5"),          # ragged unit block (12 units by 5), K tail of 64 columns
    (160, 1024, 4096, "5,7"),      # long K (16 chunks), two 80-row blocks
    (150, 64, 64, "3,2"),          # K of one box
    (136, 3072, 1024, "0,0"),      # the planner's choice
])
def test_skinny_gemm_matches_float64(M, N, K, plan, monkeypatch):
    """The skinny-M kernel (row blocks x 8-feature units over all SMs, TMA
    boxes, mma.sync, fixed-order cross-warp sums) against float64 products."""
    require_gpu()
    monkeypatch.setenv("GDIT_TEST_SKINNY", plan)
    import torch
    from flow_matching_dit_b200 import test_gemm
    g = torch.Generator().manual_seed(M * 3 + N + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16)
    bias = torch.randn(N, generator=g)
    C = test_gemm(A.cuda(), B.cuda(), bias.cuda(), bn=64, splits=1).cpu().double().numpy()
    ref = A.double().numpy() @ B.double().numpy().T + bias.double().numpy()
    np.testing.assert_allclose(C, ref, rtol=1e-5, atol=2e-5 * np.sqrt(K))


def test_gemm_rejects_bad_shapes():
    require_gpu()
    import torch
    from flow_matching_dit_b200 import GditError, test_gemm
    A = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(40, 64, dtype=torch.bfloat16, device="cuda")   # N % 32 != 0
    with pytest.raises(GditError):
        test_gemm(A, B, None)
