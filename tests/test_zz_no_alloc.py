"""The GEMM entry point that allocates nothing (gdit_gemm_static_scratch).

Some callers cannot allocate device memory while they run, for example a
robot's control loop, where cudaMalloc/cudaFree may stall the device.  This
entry point keeps its split-K scratch in a fixed array inside the library.
The test checks, through the C ABI, two calls in a row against the existing
allocating entry point (gdit_test_gemm) within the GEMM tests' tolerance, and
that sizes beyond the fixed array are rejected.  It is collected last and
holds in a fresh process as well as after the other tests.
"""

import numpy as np
import pytest

from tests.gpu_util import require_gpu

pytestmark = pytest.mark.gpu


def _inputs(M, N, K, seed):
    import torch
    g = torch.Generator().manual_seed(seed)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    B = torch.randn(N, K, generator=g).to(torch.bfloat16).cuda()
    bias = torch.randn(N, generator=g).cuda()
    return A, B, bias


@pytest.mark.parametrize("M, N, K, bn, splits, seed", [
    (17, 1024, 1024, 64, 4, 1),       # split-K: partials and tile counters in the fixed array
    (65, 512, 768, 128, 3, 2),
    (300, 1024, 512, 128, 1, 4),      # one split: the direct epilogue, no partials
])
def test_two_calls_in_a_row_match_the_allocating_entry_point(M, N, K, bn, splits, seed):
    """Two calls in a row on the same inputs: the second starts from the
    scratch contents the first left behind and must give the same result."""
    require_gpu()
    from flow_matching_dit_b200 import gemm_static_scratch, test_gemm
    A, B, bias = _inputs(M, N, K, seed)
    ref = test_gemm(A, B, bias, bn=bn, splits=splits).cpu().double().numpy()
    exact = A.cpu().double().numpy() @ B.cpu().double().numpy().T + bias.cpu().double().numpy()
    for _ in range(2):
        got = gemm_static_scratch(A, B, bias, bn=bn, splits=splits).cpu().double().numpy()
        np.testing.assert_allclose(got, ref, rtol=1e-5, atol=2e-5 * np.sqrt(K))
        np.testing.assert_allclose(got, exact, rtol=1e-5, atol=2e-5 * np.sqrt(K))


def test_sizes_beyond_the_fixed_array_are_rejected():
    require_gpu()
    from flow_matching_dit_b200 import GditError, gemm_static_scratch
    from flow_matching_dit_b200._lib import GDIT_EINVAL
    A, B, bias = _inputs(512, 4096, 512, 3)          # 4 splits x 512 x 4096 floats > 2^20
    with pytest.raises(GditError) as e:
        gemm_static_scratch(A, B, bias, bn=64, splits=4)
    assert e.value.code == GDIT_EINVAL
    A, B, bias = _inputs(128 * 65, 4096, 64, 5)      # 65 x 64 = 4160 output tiles > 4096 counters
    with pytest.raises(GditError) as e:
        gemm_static_scratch(A, B, bias, bn=64, splits=1)
    assert e.value.code == GDIT_EINVAL
