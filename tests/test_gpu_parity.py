"""GPU parity of the CUDA path against the fp64 oracle (run on a B200).

Tolerances (from the solver's acceptance rule):
* codes identical to the oracle on the 64x128 workloads and on small ragged shapes;
* elsewhere the codes satisfy the closed-form fixed point W = Q(W* + (I+L_O)^T E (I+L_I) - E)
  evaluated in fp64, except entries whose pre/s lies within 1e-3 grid steps of a rounding
  boundary, and such exempt mismatches are at most 0.1% of the entries;
* the proxy loss within 1e-3 relative of the fp64 value.
Every parity call goes through the C ABI (ctypes binding).
"""
import os
import subprocess
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import (band_check, code_range, fixed_point_pre, fixed_point_pre_rows, proxy_loss,
                    round_naive, round_row_sweep, udu)
from two_sided_adaptive_bakron_b200.workloads import make_workload, random_problem

from ._helpers import cond_estimate, library_udu, library_udu_torch

pytestmark = pytest.mark.gpu

BAND = 1e-3
MAX_EXEMPT_FRAC = 1e-3


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


def _gpu_round(bk, Ws, LO32, LI32, s, bits):
    codes, W = bk.round_weights(_dev(Ws), _dev(LO32), _dev(LI32), _dev(s), bits)
    return codes.cpu().numpy().astype(np.int64), W.cpu().numpy()


def _oracle_factors32(HO, HI):
    LO, _ = udu(HO)
    LI, _ = udu(HI)
    return LO.astype(np.float32), LI.astype(np.float32)


# ----------------------------------------------------------------------------- round: exact
@pytest.mark.parametrize("name", ["small_64x128", "small_64x128_ho_identity",
                                  "small_64x128_identity"])
def test_round_codes_identical_to_oracle_small(bk, name):
    Ws, HO, HI, s, bits = make_workload(name)
    LO32, LI32 = _oracle_factors32(HO, HI)
    C_ref, W_ref = round_naive(Ws, LO32, LI32, s, bits)
    C, W = _gpu_round(bk, Ws, LO32, LI32, s, bits)
    np.testing.assert_array_equal(C, C_ref)
    np.testing.assert_array_equal(W, (s[:, None] * C.astype(np.float32)).astype(np.float32))


@pytest.mark.parametrize("m,n,bits,seed", [(1, 1, 2, 0), (1, 70, 3, 1), (70, 1, 2, 2),
                                           (7, 300, 2, 3), (33, 65, 4, 4), (64, 31, 2, 5),
                                           (100, 37, 3, 6), (31, 33, 8, 7), (96, 96, 2, 8),
                                           # several super-blocks (far-field pushes) with partial
                                           # leaves and tiles: row strides that allow tensor box
                                           # loads (multiples of 4) and ones that do not
                                           (520, 780, 3, 9), (515, 777, 3, 10)])
def test_round_codes_identical_ragged(bk, m, n, bits, seed):
    Ws, HO, HI, s, _ = random_problem(m, n, bits, seed)
    LO32, LI32 = _oracle_factors32(HO, HI)
    C_ref, _ = round_row_sweep(Ws, LO32, LI32, s, bits)
    C, _ = _gpu_round(bk, Ws, LO32, LI32, s, bits)
    np.testing.assert_array_equal(C, C_ref)


def test_round_zero_scale_row(bk):
    Ws, HO, HI, s, bits = random_problem(40, 50, 2, 11)
    Ws[5] = 0.0
    s = s.copy()
    s[5] = 0.0
    LO32, LI32 = _oracle_factors32(HO, HI)
    C_ref, _ = round_row_sweep(Ws, LO32, LI32, s, bits)
    C, W = _gpu_round(bk, Ws, LO32, LI32, s, bits)
    np.testing.assert_array_equal(C, C_ref)
    assert np.all(W[5] == 0)


def test_round_deterministic(bk):
    Ws, HO, HI, s, bits = make_workload("sq_1024")
    LO, _ = library_udu(HO)
    LI, _ = library_udu(HI)
    a = _gpu_round(bk, Ws, LO.astype(np.float32), LI.astype(np.float32), s, bits)
    b = _gpu_round(bk, Ws, LO.astype(np.float32), LI.astype(np.float32), s, bits)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


# ----------------------------------------------------------------------------- round: fixed point
def test_round_fixed_point_sq_1024_full(bk):
    Ws, HO, HI, s, bits = make_workload("sq_1024")
    LO, _ = library_udu(HO)
    LI, _ = library_udu(HI)
    LO32, LI32 = LO.astype(np.float32), LI.astype(np.float32)
    C, W = _gpu_round(bk, Ws, LO32, LI32, s, bits)
    pre = fixed_point_pre(Ws, W, LO32, LI32)
    mism, outside, in_band = band_check(pre, C, s, bits, BAND)
    assert outside == 0, (mism, outside, in_band)
    assert mism <= MAX_EXEMPT_FRAC * C.size


@pytest.mark.parametrize("name", ["attn_4096", "down_4096x14336", "upgate_28672x8192"])
def test_round_fixed_point_full_size_sampled_rows(bk, name):
    Ws, HO, HI, s, bits = make_workload(name, device="cuda")
    m, n = Ws.shape
    LO32, _ = library_udu_torch(HO, "cuda")
    LI32, _ = library_udu_torch(HI, "cuda")
    C, W = _gpu_round(bk, Ws, LO32, LI32, s, bits)
    rng = np.random.default_rng(123)
    rows = np.unique(np.concatenate([[0, 1, 31, 32, m - 1], rng.integers(0, m, 11)]))
    pre = fixed_point_pre_rows(Ws, W, LO32, LI32, rows)
    mism, outside, in_band = band_check(pre, C[rows], s[rows], bits, BAND)
    assert outside == 0, (mism, outside, in_band)
    assert mism <= max(1, MAX_EXEMPT_FRAC * pre.size)
    lo, hi = code_range(bits)
    assert C.min() >= lo and C.max() <= hi


# ----------------------------------------------------------------------------- ldl
@pytest.mark.parametrize("d,seed", [(1, 0), (5, 1), (31, 2), (32, 3), (33, 4), (100, 5),
                                    (257, 6), (1024, 7),
                                    # the look-ahead path (two plane sets, side stream), with
                                    # partial outer and inner blocks
                                    (2049, 8), (3001, 9), (4096, 10)])
def test_ldl_matches_oracle(bk, d, seed):
    _, H, _, _, _ = random_problem(d, 3, 2, seed)
    L, D = bk.ldl(_dev(H))
    L, D = L.cpu().numpy().astype(np.float64), D.cpu().numpy().astype(np.float64)
    assert np.all(np.tril(L) == 0)
    L_ref, D_ref = udu(H) if d <= 300 else library_udu(H)
    U = np.eye(d) + L
    rec = U @ np.diag(D) @ U.T
    H64 = H.astype(np.float64)
    # backward error of an fp32 factorisation: a small multiple of d * eps32 * |H|
    assert np.abs(rec - H64).max() <= 4 * d * 6e-8 * np.abs(H64).max() + 1e-30
    # forward error, scaled by the conditioning of the factor
    kappa = np.linalg.cond(H64) if d <= 1024 else cond_estimate(H64, "cuda")
    tol = 50 * kappa * 6e-8 * max(1.0, np.abs(L_ref).max())
    assert np.abs(L - L_ref).max() <= tol
    np.testing.assert_allclose(D, D_ref, rtol=50 * kappa * 6e-8)


def test_ldl_rejects_indefinite(bk):
    H = np.eye(40, dtype=np.float32)
    H[3, 3] = -1.0
    st = bk.new_status("cuda")
    L = torch.empty((40, 40), device="cuda")
    D = torch.empty(40, device="cuda")
    ws = bk.workspace(bk.bakron_ldl_workspace_bytes(40), "cuda")
    assert bk.bakron_ldl(_dev(H), L, D, ws, st) == 0
    assert bk.bakron_read_status(st) == bk.BAKRON_ERR_NOT_PD


# ----------------------------------------------------------------------------- proxy loss
@pytest.mark.parametrize("m,n,seed", [(1, 1, 0), (3, 70, 1), (64, 128, 2), (200, 130, 3),
                                      (513, 257, 4)])
def test_proxy_loss_random(bk, m, n, seed):
    _, HO, HI, _, _ = random_problem(m, n, 2, seed)
    dW = np.random.default_rng(seed).standard_normal((m, n)).astype(np.float32)
    got = float(bk.proxy_loss(_dev(dW), _dev(HO), _dev(HI)).item())
    ref = proxy_loss(dW, HO, HI)
    assert abs(got - ref) <= 1e-3 * abs(ref)


@pytest.mark.parametrize("name", ["small_64x128", "sq_1024"])
def test_proxy_loss_of_rounding_residual(bk, name):
    Ws, HO, HI, s, bits = make_workload(name)
    LO, _ = library_udu(HO)
    LI, _ = library_udu(HI)
    C, W = _gpu_round(bk, Ws, LO.astype(np.float32), LI.astype(np.float32), s, bits)
    dW = (Ws - W).astype(np.float32)
    got = float(bk.proxy_loss(_dev(dW), _dev(HO), _dev(HI)).item())
    ref = proxy_loss(dW, HO, HI)
    assert abs(got - ref) <= 1e-3 * abs(ref), (got, ref)


def test_whole_path_small(bk):
    Ws, HO, HI, s, bits = make_workload("small_64x128")
    codes, W, loss, (LO, DO), (LI, DI) = bk.solve(_dev(Ws), _dev(HO), _dev(HI), _dev(s), bits)
    LO, LI = LO.cpu().numpy(), LI.cpu().numpy()
    C = codes.cpu().numpy().astype(np.int64)
    Wn = W.cpu().numpy()
    pre = fixed_point_pre(Ws, Wn, LO, LI)
    mism, outside, _ = band_check(pre, C, s, bits, BAND)
    assert outside == 0
    ref = proxy_loss(Ws - Wn, HO, HI)
    assert abs(float(loss.item()) - ref) <= 1e-3 * ref


# ----------------------------------------------------------------------------- fault paths
def test_nonfinite_input_reported(bk):
    Ws, HO, HI, s, bits = random_problem(40, 40, 2, 3)
    Ws[7, 9] = np.nan
    LO32, LI32 = _oracle_factors32(HO, HI)
    with pytest.raises(bk.BakronError) as ei:
        bk.round_weights(_dev(Ws), _dev(LO32), _dev(LI32), _dev(s), bits)
    assert ei.value.code == bk.BAKRON_ERR_NONFINITE


def test_dependency_wait_timeout_is_reported_not_hung(bk):
    """A 1 ns wait limit makes every dependency wait that is not already satisfied give up:
    the launch must end with BAKRON_ERR_TIMEOUT and leave the context usable."""
    code = r"""
import numpy as np, torch
from two_sided_adaptive_bakron_b200 import bakron as bk
from two_sided_adaptive_bakron_b200.workloads import random_problem
Ws, HO, HI, s, bits = random_problem(512, 512, 2, 1)
L = np.triu(np.full((512, 512), 0.001, np.float32), 1)
st = bk.new_status('cuda')
codes = torch.empty((512, 512), dtype=torch.int8, device='cuda')
W = torch.empty((512, 512), device='cuda')
ws = bk.workspace(bk.bakron_round_workspace_bytes(512, 512), 'cuda')
d = lambda x: torch.from_numpy(x).cuda()
rc = bk.bakron_round(d(Ws), d(L), d(L), d(s), bits, codes, W, ws, st)
print('RC', rc, 'STATUS', bk.bakron_read_status(st))
x = torch.ones(10, device='cuda').sum().item()
print('ALIVE', x)
"""
    env = dict(os.environ, BAKRON_SPIN_LIMIT_NS="1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], env=env, cwd=root, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert "RC 0 STATUS -4" in r.stdout, r.stdout
    assert "ALIVE 10.0" in r.stdout
