"""GPU parity of the incoherence-processing kernels (bakron_rht, bakron_row_scales) and of the
rotated solve, against the fp64 oracle (run on a B200), through the C ABI.

* A one-entry input makes every butterfly and order-28 sum add zeros, so the output is exact:
  every entry is +-fl(fl(1/sqrt(c)) fl(1/sqrt(r))) with the sign of T_r[k, i] T_c[l, j]. The sign
  pattern and the magnitude are compared exactly (all index and sign logic of both passes).
* Random inputs: relative Frobenius error at most 2e-5 against the oracle. The bound is the
  worst case of the arithmetic: each butterfly level adds at most sqrt(2) u of the norm
  (u = 2^-24), an order-28 sum at most 27 sqrt(28) u of its inputs' norm, over both sides.
  Rows of 28 * 2^k >= 1792 form the order-28 sums on the tensor cores: the data split hi + lo
  (lo truncated to tf32: at most 2^-21 of the value), 56 terms accumulated in fp32 without
  round-to-nearest (at most 2^-23 of the running sum each), about 7e-6 of the inputs' norm;
  typical errors are near 1e-7.
* Full size (the 4096 x 14336 and 28672 x 8192 layers, and shapes that reach the row lengths
  2048, 16384 and 32768): sampled entries against the oracle's rows of T, the round trip and
  the norm.
* Grid steps: bitwise equal to fp32 max / divisor.
* The rotated solve: the proxy loss in the rotated basis equals the oracle's loss of the
  unrotated weights in the original basis, W_orig = T_m^T W~_q T_n, and the rotated codes are a
  fixed point of the rule under the band rule.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import (band_check, fixed_point_pre, hadamard_rows, proxy_loss, rht, rht_signs)
from two_sided_adaptive_bakron_b200.workloads import make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from two_sided_adaptive_bakron_b200 import build
    build.build()
    from two_sided_adaptive_bakron_b200 import bakron
    return bakron


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def _t_rows(d, seed, idx):
    return hadamard_rows(d, idx) * rht_signs(d, seed)[None, :] / np.sqrt(d)


@pytest.mark.parametrize("r,c,i,j,inverse", [(1, 1, 0, 0, 0), (2, 28, 1, 27, 0),
                                             (28, 4, 13, 2, 1), (56, 64, 55, 0, 0),
                                             (112, 448, 77, 300, 1), (64, 896, 5, 895, 0),
                                             (4, 1792, 3, 1000, 0), (2, 3584, 1, 3583, 1)])
def test_spike_is_exact(bk, r, c, i, j, inverse):
    X = np.zeros((r, c), dtype=np.float32)
    X[i, j] = 1.0
    sr, sc = 101, 202
    Y = bk.rht(_dev(X), sr, sc, inverse=bool(inverse)).cpu().numpy()
    ref = rht(X, sr, sc, inverse=bool(inverse))
    mag = np.float32(np.float32(1.0) / np.sqrt(np.float32(c))) * \
        np.float32(np.float32(1.0) / np.sqrt(np.float32(r)))
    np.testing.assert_array_equal(np.abs(Y), np.full((r, c), mag, dtype=np.float32))
    np.testing.assert_array_equal(np.sign(Y), np.sign(ref))


@pytest.mark.parametrize("r,c,inverse", [(1, 28, 0), (28, 28, 1), (64, 112, 0), (448, 32, 1),
                                         (1024, 224, 0), (128, 128, 1), (28, 1792, 1),
                                         (8, 3584, 0)])
def test_random_matches_oracle(bk, r, c, inverse):
    X = np.random.default_rng(r * 7 + c).standard_normal((r, c)).astype(np.float32)
    Y = bk.rht(_dev(X), 5, 6, inverse=bool(inverse)).cpu().numpy().astype(np.float64)
    ref = rht(X, 5, 6, inverse=bool(inverse))
    assert np.linalg.norm(Y - ref) <= 2e-5 * np.linalg.norm(ref)


def test_in_place(bk):
    X = np.random.default_rng(3).standard_normal((56, 64)).astype(np.float32)
    d = _dev(X)
    ws = bk.workspace(bk.bakron_rht_workspace_bytes(56, 64), "cuda")
    assert bk.bakron_rht(d, 9, 10, False, d, ws) == 0
    np.testing.assert_array_equal(d.cpu().numpy(), bk.rht(_dev(X), 9, 10).cpu().numpy())


# the layer shapes of the benchmark workloads (4096 x 14336, 28672 x 8192) and the row
# lengths that no smaller test reaches: 2048, 8192, 16384, 28672 and 32768
@pytest.mark.parametrize("r,c", [(4096, 14336), (28672, 8192), (2048, 16384), (512, 32768)])
def test_full_size_sampled_and_round_trip(bk, r, c):
    X = np.random.default_rng(11).standard_normal((r, c)).astype(np.float32)
    Xd = _dev(X)
    Y = bk.rht(Xd, 12, 13)
    back = bk.rht(Y, 12, 13, inverse=True)
    nx = float(torch.linalg.norm(Xd.double()))
    assert float(torch.linalg.norm(back.double() - Xd.double())) <= 4e-5 * nx
    assert abs(float(torch.linalg.norm(Y.double())) - nx) <= 2e-5 * nx
    rows = np.unique(np.array([0, 1, r // 2 - 1, r // 2, r - 1]))
    cols = np.unique(np.array([0, c // 28 - 1, c // 28, c // 2, c - 1]))
    Tr = _t_rows(r, 12, rows)
    Tc = _t_rows(c, 13, cols)
    ref = Tr @ X.astype(np.float64) @ Tc.T
    got = Y.cpu().numpy()[np.ix_(rows, cols)]
    assert np.abs(got - ref).max() <= 1e-4


# column lengths that select the column passes' remaining variants: 28 2^k with 2^k between 32
# and 512 (896), 2^k above 4096 (8192, 16384, 32768: up to 64 rows per thread in the strided
# pass) and 28 * 512 (14336: order-28 stage alone in the strided pass)
@pytest.mark.parametrize("r,c", [(896, 64), (8192, 32), (14336, 28), (16384, 28), (32768, 32)])
def test_column_lengths_sampled_and_round_trip(bk, r, c):
    X = np.random.default_rng(r + c).standard_normal((r, c)).astype(np.float32)
    Xd = _dev(X)
    Y = bk.rht(Xd, 21, 22)
    back = bk.rht(Y, 21, 22, inverse=True)
    nx = float(torch.linalg.norm(Xd.double()))
    assert float(torch.linalg.norm(back.double() - Xd.double())) <= 4e-5 * nx
    assert abs(float(torch.linalg.norm(Y.double())) - nx) <= 2e-5 * nx
    rows = np.unique(np.array([0, 1, 511, 512, r // 28, r // 2, r - 1]))
    cols = np.arange(c)
    ref = _t_rows(r, 21, rows) @ X.astype(np.float64) @ _t_rows(c, 22, cols).T
    got = Y.cpu().numpy()[np.ix_(rows, cols)]
    assert np.abs(got - ref).max() <= 1e-4


# row lengths 28 S (S = 256, 512, 1024) of the tensor-core row pass, both directions (the
# inverse through the round trip), on a few rows; sampled columns across segment boundaries
@pytest.mark.parametrize("r,c", [(8, 7168), (16, 14336), (4, 28672)])
def test_row_lengths_sampled_and_round_trip(bk, r, c):
    X = np.random.default_rng(r + c).standard_normal((r, c)).astype(np.float32)
    Xd = _dev(X)
    Y = bk.rht(Xd, 31, 32)
    back = bk.rht(Y, 31, 32, inverse=True)
    nx = float(torch.linalg.norm(Xd.double()))
    assert float(torch.linalg.norm(back.double() - Xd.double())) <= 4e-5 * nx
    assert abs(float(torch.linalg.norm(Y.double())) - nx) <= 2e-5 * nx
    S = c // 28
    cols = np.unique(np.array([0, 1, 7, 8, 31, 32, S - 1, S, 5 * S + 17, c // 2, c - 2, c - 1]))
    ref = _t_rows(r, 31, np.arange(r)) @ X.astype(np.float64) @ _t_rows(c, 32, cols).T
    got = Y.cpu().numpy()[:, cols]
    assert np.abs(got - ref).max() <= 1e-4


@pytest.mark.parametrize("m,n,group,div", [(5, 37, 37, 1.5), (64, 128, 32, 3.5), (3, 100, 7, 1.0)])
def test_row_scales_exact(bk, m, n, group, div):
    W = np.random.default_rng(m + n).standard_normal((m, n)).astype(np.float32)
    G = (n + group - 1) // group
    ref = np.stack([np.abs(W[:, g * group:(g + 1) * group]).max(axis=1) for g in range(G)],
                   axis=1) / np.float32(div)
    got = bk.row_scales(_dev(W), div, group_size=group).cpu().numpy()
    np.testing.assert_array_equal(got, ref.astype(np.float32))


def test_rotated_solve(bk):
    Ws, HO, HI, s, bits = make_workload("small_64x128")
    solver = bk.Solver(64, 128, "cuda")
    so, si = 31, 32
    solver.run(_dev(Ws), _dev(HO), _dev(HI), None, bits, incoherence=(so, si))
    solver.check()
    Wq_rot = solver.W.cpu().numpy().astype(np.float64)
    W_orig = solver.W_orig.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(W_orig, rht(Wq_rot, so, si, inverse=True), rtol=0, atol=1e-5)
    ref = proxy_loss(Ws.astype(np.float64) - W_orig, HO, HI)
    assert abs(float(solver.loss.item()) - ref) <= 1e-3 * ref
    # the rotated codes satisfy the rule on the rotated layer (the solver's own factors)
    Wt = rht(Ws, so, si).astype(np.float32)
    st = (np.abs(Wt).max(axis=1) / np.float32((1 << (bits - 1)) - 0.5)).astype(np.float32)
    pre = fixed_point_pre(Wt, Wq_rot, solver.L_O.cpu().numpy(), solver.L_I.cpu().numpy())
    mism, outside, _ = band_check(pre, solver.codes.cpu().numpy().astype(np.int64), st, bits,
                                  1e-3)
    assert outside == 0 and mism <= 0.001 * Ws.size
