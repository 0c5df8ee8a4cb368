"""GPU parity of the Kronecker-factor kernels (bakron_damped_gram, bakron_sketch_b) against the
fp64 oracle (run on a B200), through the C ABI.

Tolerance: every entry within tol(K) sqrt(H_aa H_bb) of the oracle, sqrt(H_aa H_bb) being the
Cauchy-Schwarz bound on the mean |x_a x_b| (the scale of the sum). The products run as
3xTF32: hi = the tf32 truncation of x, lo = x - hi read as tf32, hi*hi + hi*lo + lo*hi, so each
product is within 3 * 2^-20 of exact. The tensor core's fp32 accumulator does not round to
nearest (measured on B200 at about half an ulp, 2^-23, of the running sum lost per MMA
instruction), so the library restarts it every 256 samples: one chunk takes at most
3 * 256 / 8 = 96 instructions (three passes of depth-8 tf32 MMAs), and the ceil(K / 256) chunk
sums are added in round-to-nearest fp32, at most 2^-24 of the running sum each. With two ulps
allowed per instruction:
    tol(K) = (3 min(K, 256) / 8 + 2) 2^-22 + ceil(K / 256) 2^-24 + 3 * 2^-20,
about 2.8e-5 at K = 8192 (it would be 7.3e-4 with one accumulator over all of K). A dropped lo
pass (error about 2^-10) fails it at every K. The result must be exactly symmetric.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import (band_check, damped_gram, damped_gram_rows, fixed_point_pre, proxy_loss,
                    sketch_b)
from two_sided_adaptive_bakron_b200.workloads import make_layer_samples

pytestmark = pytest.mark.gpu


def tol(K):
    return ((3 * min(K, 256) / 8 + 2) * 2.0 ** -22 + -(-K // 256) * 2.0 ** -24
            + 3 * 2.0 ** -20)


@pytest.fixture(scope="module")
def bk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from two_sided_adaptive_bakron_b200 import build
    build.build()
    from two_sided_adaptive_bakron_b200 import bakron
    return bakron


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _check(H, H_ref, diag_rows, diag_cols, K):
    bound = tol(K) * np.sqrt(np.outer(np.abs(diag_rows), np.abs(diag_cols)))
    err = np.abs(H.astype(np.float64) - H_ref)
    worst = float((err / bound).max())
    assert worst <= 1.0, worst


@pytest.mark.parametrize("N,d,seed", [(1, 1, 0), (5, 3, 1), (100, 129, 2), (257, 300, 3),
                                      (1000, 640, 4), (2048, 1024, 5), (33, 2000, 6),
                                      (8229, 384, 7)])
def test_damped_gram_matches_oracle(bk, N, d, seed):
    rng = np.random.default_rng(seed)
    X = (rng.standard_normal((N, d)) * np.exp(rng.standard_normal(d))[None, :]).astype(np.float32)
    H = bk.damped_gram(_dev(X), 0.01)
    assert torch.equal(H, H.T)
    H = H.cpu().numpy()
    ref = damped_gram(X, 0.01)
    _check(H, ref, np.diag(ref), np.diag(ref), N)


def test_damped_gram_damping_and_zero_columns(bk):
    X = np.random.default_rng(7).standard_normal((64, 48)).astype(np.float32)
    X[:, 5] = 0.0
    H0 = bk.damped_gram(_dev(X), 0.0).cpu().numpy()
    H1 = bk.damped_gram(_dev(X), 0.5).cpu().numpy()
    off = ~np.eye(48, dtype=bool)
    np.testing.assert_array_equal(H0[off], H1[off])
    assert np.all(H0[5] == 0) and np.all(H0[:, 5] == 0)
    mean = np.mean(np.diag(H0).astype(np.float64))
    np.testing.assert_allclose(np.diag(H1) - np.diag(H0), 0.5 * mean, rtol=1e-5)


def test_damped_gram_full_size_sampled_rows(bk):
    # the 4096 x 14336 layer's samples: X (8192 tokens x 14336) for H_I, G (8192 x 4096) for H_O
    _, X, G, _, _ = make_layer_samples("down_4096x14336")
    rng = np.random.default_rng(11)
    for A in (X, G):
        N, d = A.shape
        H = bk.damped_gram(_dev(A), 0.01)
        assert torch.equal(H, H.T)
        rows = np.unique(np.concatenate([[0, 1, 127, 128, d - 1], rng.integers(0, d, 5)]))
        Hr = H[torch.from_numpy(rows).cuda()].cpu().numpy()
        del H
        torch.cuda.empty_cache()
        ref = damped_gram_rows(A, 0.01, rows)
        diag = np.einsum("ti,ti->i", A.astype(np.float64), A.astype(np.float64)) / N
        diag += 0.01 * diag.mean()
        _check(Hr, ref, diag[rows], diag, N)


@pytest.mark.parametrize("S,m,n,seed", [(1, 1, 1, 0), (3, 5, 7, 1), (4, 70, 130, 2),
                                        (8, 128, 256, 3), (16, 300, 200, 4), (5, 513, 257, 5)])
def test_sketch_b_matches_oracle(bk, S, m, n, seed):
    G = np.random.default_rng(seed).standard_normal((S, m, n)).astype(np.float32)
    H_O, H_I = bk.sketch_b(_dev(G), 0.01)
    assert torch.equal(H_O, H_O.T) and torch.equal(H_I, H_I.T)
    HO_ref, HI_ref = sketch_b(G, 0.01)
    _check(H_O.cpu().numpy(), HO_ref, np.diag(HO_ref), np.diag(HO_ref), S * n)
    _check(H_I.cpu().numpy(), HI_ref, np.diag(HI_ref), np.diag(HI_ref), S * m)


def test_sketch_b_factors_feed_the_solver(bk):
    # the factors go straight into the factorisation and the round (whole path on the device)
    S, m, n, bits = 16, 64, 96, 3
    G = np.random.default_rng(9).standard_normal((S, m, n)).astype(np.float32)
    H_O, H_I = bk.sketch_b(_dev(G), 0.01)
    Ws = (np.random.default_rng(10).standard_normal((m, n)) / np.sqrt(n)).astype(np.float32)
    s = (np.abs(Ws).max(axis=1) / np.float32((1 << (bits - 1)) - 0.5)).astype(np.float32)
    codes, W, loss, (L_O, _), (L_I, _) = bk.solve(_dev(Ws), H_O, H_I, _dev(s), bits)
    lo, hi = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
    c = codes.cpu().numpy().astype(np.int64)
    assert c.min() >= lo and c.max() <= hi
    # the codes are the rule's fixed point with the factors the library made of these factors
    Wn = W.cpu().numpy()
    pre = fixed_point_pre(Ws, Wn, L_O.cpu().numpy(), L_I.cpu().numpy())
    mism, outside, _ = band_check(pre, c, s, bits, 1e-3)
    assert outside == 0 and mism <= 1e-3 * c.size
    # and the loss is that of the residual under the Sketch-B factors themselves
    ref = proxy_loss(Ws - Wn, H_O.cpu().numpy(), H_I.cpu().numpy())
    assert abs(float(loss.item()) - ref) <= 1e-3 * ref


def test_invalid_arguments(bk):
    X = torch.zeros((4, 4), device="cuda")
    H = torch.zeros((4, 4), device="cuda")
    ws = bk.workspace(bk.bakron_damped_gram_workspace_bytes(4, 4), "cuda")
    st = bk.new_status("cuda")
    assert bk.bakron_damped_gram(X, -1.0, H, ws, st) == bk.BAKRON_ERR_INVALID_ARG
    small = bk.workspace(256, "cuda")
    assert bk.bakron_damped_gram(X, 0.01, H, small, st) == bk.BAKRON_ERR_WORKSPACE
