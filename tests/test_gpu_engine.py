"""GPU checks of the 3xTF32 tensor-core GEMM engine (tcgen05 + TMA + TMEM) in isolation,
against fp64 products computed on the host."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from two_sided_adaptive_bakron_b200 import build
    build.build()
    from two_sided_adaptive_bakron_b200 import bakron
    return bakron


@pytest.mark.parametrize("M,N,K,seed", [(128, 128, 32, 0), (128, 128, 256, 1), (256, 384, 1024, 2),
                                        (100, 37, 50, 3), (1, 1, 1, 4), (130, 129, 33, 5),
                                        (640, 256, 4096, 6)])
def test_gemm3x_matches_fp64(bk, M, N, K, seed):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((M, K)).astype(np.float32)
    B = rng.standard_normal((N, K)).astype(np.float32)
    C = bk.internal_gemm3x(torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda()).cpu().numpy()
    ref = A.astype(np.float64) @ B.astype(np.float64).T
    mag = np.abs(A).astype(np.float64) @ np.abs(B).astype(np.float64).T
    # 3xTF32: ~2^-21 relative per product plus fp32 accumulation
    err = np.abs(C - ref)
    assert np.all(err <= 4e-6 * mag + 1e-30), float((err / (mag + 1e-30)).max())


def test_gemm3x_beats_single_tf32_precision(bk):
    """The hi/lo terms are really used: the error is far below what one tf32 pass gives."""
    rng = np.random.default_rng(9)
    A = rng.standard_normal((256, 512)).astype(np.float32)
    B = rng.standard_normal((256, 512)).astype(np.float32)
    C = bk.internal_gemm3x(torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda()).cpu().numpy()
    ref = A.astype(np.float64) @ B.astype(np.float64).T
    mag = np.abs(A).astype(np.float64) @ np.abs(B).astype(np.float64).T
    rel = float((np.abs(C - ref) / mag).max())
    assert rel < 2e-6, rel


@pytest.mark.parametrize("m,n,seed", [(64, 128, 0), (300, 200, 1), (1000, 1500, 2)])
def test_tensor_core_loss_matches_cuda_core_loss(bk, m, n, seed):
    from two_sided_adaptive_bakron_b200.workloads import random_problem
    _, HO, HI, _, _ = random_problem(m, n, 2, seed)
    dW = np.random.default_rng(seed).standard_normal((m, n)).astype(np.float32)
    d = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    a = float(bk.proxy_loss(d(dW), d(HO), d(HI)).item())
    b = float(bk.internal_proxy_loss_simt(d(dW), d(HO), d(HI)).item())
    assert abs(a - b) <= 1e-4 * abs(b)
