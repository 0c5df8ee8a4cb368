"""GPU parity of bakron_round_ex (per-group grid steps, scalar codebooks) against the fp64
oracle (run on a B200), through the C ABI.

Tolerances are those of the nearest-rounding parity tests, the rounding boundaries being the
half-integers (integer grid) or the codebook midpoints: codes identical to the oracle on small
shapes; on larger shapes identical, or else the GPU result is a fixed point of the closed form
W = Q(W* + (I+L_O)^T E (I+L_I) - E) except entries within 1e-3 grid steps of a boundary, at
most 0.1% of them.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import (band_check, code_range, fixed_point_pre, fixed_point_pre_rows,
                    round_naive, round_row_sweep, udu)
from two_sided_adaptive_bakron_b200.workloads import make_workload, random_problem

from ._helpers import library_udu_torch

pytestmark = pytest.mark.gpu

BAND = 1e-3
MAX_EXEMPT_FRAC = 1e-3
CB3 = np.array([-1.0, -0.62, -0.33, -0.1, 0.08, 0.3, 0.61, 1.0], dtype=np.float32)


def _codebook(bits):
    """Normal quantiles (k + 1/2) / K mapped to [-1, 1]: a non-uniform, symmetric codebook."""
    from statistics import NormalDist
    K = 1 << bits
    q = np.array([NormalDist().inv_cdf((k + 0.5) / K) for k in range(K)])
    return (q / np.abs(q).max()).astype(np.float32)


def _group_scales(Ws, gs, top):
    m, n = Ws.shape
    G = (n + gs - 1) // gs
    s = np.zeros((m, G), dtype=np.float32)
    for g in range(G):
        s[:, g] = np.abs(Ws[:, g * gs:(g + 1) * gs]).max(axis=1) / np.float32(top)
    return s


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


def _gpu(bk, Ws, LO, LI, s, bits, gs, cb):
    codes, W = bk.round_weights(_dev(Ws), _dev(LO), _dev(LI), _dev(s), bits, group_size=gs,
                                codebook=cb)
    return codes.cpu().numpy().astype(np.int64), W.cpu().numpy()


def _factors32(HO, HI):
    return udu(HO)[0].astype(np.float32), udu(HI)[0].astype(np.float32)


@pytest.mark.parametrize("name", ["small_64x128", "small_64x128_identity"])
@pytest.mark.parametrize("gs,bits,cb", [(32, 3, "cb3"), (128, 4, "normal"), (64, 4, None),
                                        (1 << 20, 2, "normal"), (32, 1, "normal")])
def test_codes_identical_small(bk, name, gs, bits, cb):
    Ws, HO, HI, _, _ = make_workload(name)
    LO, LI = _factors32(HO, HI)
    book = CB3 if cb == "cb3" else (_codebook(bits) if cb else None)
    g = min(gs, Ws.shape[1])
    s = _group_scales(Ws, g, 1.0 if book is not None else (1 << (bits - 1)) - 0.5)
    C_ref, W_ref = round_naive(Ws, LO, LI, s, bits, codebook=book, group_size=g)
    C, W = _gpu(bk, Ws, LO, LI, s, bits, gs, book)
    np.testing.assert_array_equal(C, C_ref)
    sfull = np.repeat(s, g, axis=1)[:, :Ws.shape[1]]
    vals = C.astype(np.float32) if book is None else book[C]
    np.testing.assert_array_equal(W, (sfull * vals).astype(np.float32))


@pytest.mark.parametrize("m,n,bits,gs,cb,seed", [(1, 1, 2, 32, "normal", 0), (7, 300, 3, 64, "cb3", 1),
                                                 (33, 65, 4, 32, "normal", 2), (100, 37, 3, 32, None, 3),
                                                 (96, 96, 2, 64, "normal", 4),
                                                 (520, 780, 3, 128, "cb3", 5),
                                                 (515, 777, 4, 96, "normal", 6)])
def test_ragged(bk, m, n, bits, gs, cb, seed):
    Ws, HO, HI, _, _ = random_problem(m, n, bits, seed + 70)
    LO, LI = _factors32(HO, HI)
    book = CB3 if cb == "cb3" else (_codebook(bits) if cb else None)
    g = min(gs, n)
    s = _group_scales(Ws, g, 1.0 if book is not None else (1 << (bits - 1)) - 0.5)
    C_ref, _ = round_row_sweep(Ws, LO, LI, s, bits, codebook=book, group_size=g)
    C, W = _gpu(bk, Ws, LO, LI, s, bits, gs, book)
    if m * n <= 20000 or np.array_equal(C, C_ref):
        np.testing.assert_array_equal(C, C_ref)
        return
    pre = fixed_point_pre(Ws, W, LO, LI)
    mism, outside, in_band = band_check(pre, C, s, bits, BAND, codebook=book, group_size=g)
    assert outside == 0, (mism, outside, in_band)
    assert mism <= MAX_EXEMPT_FRAC * C.size


def test_one_group_equals_bakron_round(bk):
    Ws, HO, HI, s, bits = make_workload("sq_1024")
    LO, _ = library_udu_torch(HO, "cuda")
    LI, _ = library_udu_torch(HI, "cuda")
    a = bk.round_weights(_dev(Ws), _dev(LO), _dev(LI), _dev(s), bits)
    b = bk.round_weights(_dev(Ws), _dev(LO), _dev(LI), _dev(s[:, None]), bits, group_size=1024)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_full_size_sampled_rows(bk):
    Ws, HO, HI, _, _ = make_workload("down_4096x14336", device="cuda")
    m, n = Ws.shape
    bits, gs, book = 3, 128, _codebook(3)
    s = _group_scales(Ws, gs, 1.0)
    LO, _ = library_udu_torch(HO, "cuda")
    LI, _ = library_udu_torch(HI, "cuda")
    C, W = _gpu(bk, Ws, LO, LI, s, bits, gs, book)
    rows = np.unique(np.concatenate([[0, 1, 31, 32, m - 1],
                                     np.random.default_rng(5).integers(0, m, 6)]))
    pre = fixed_point_pre_rows(Ws, W, LO, LI, rows)
    mism, outside, in_band = band_check(pre, C[rows], s[rows], bits, BAND, codebook=book,
                                        group_size=gs)
    assert outside == 0, (mism, outside, in_band)
    assert mism <= max(1, MAX_EXEMPT_FRAC * pre.size)
    assert C.min() >= 0 and C.max() <= 7


def test_invalid_quantizers_rejected(bk):
    m, n = 8, 64
    Ws = torch.zeros((m, n), device="cuda")
    L = torch.zeros((m, m), device="cuda")
    LI = torch.zeros((n, n), device="cuda")
    codes = torch.empty((m, n), dtype=torch.int8, device="cuda")
    W = torch.empty((m, n), device="cuda")
    ws = bk.workspace(bk.bakron_round_workspace_bytes(m, n), "cuda")
    st = bk.new_status("cuda")
    s2 = torch.ones((m, 2), device="cuda")
    E = bk.BAKRON_ERR_INVALID_ARG
    # group size not a multiple of the leaf width
    assert bk.bakron_round_ex(Ws, L, LI, torch.ones((m, 2), device="cuda"), 48, None, 3, codes, W,
                              ws, st) == E
    # codebook not increasing, not finite, too many entries
    assert bk.bakron_round_ex(Ws, L, LI, s2, 32, [0.0, 1.0, 0.5, 2.0], 2, codes, W, ws, st) == E
    assert bk.bakron_round_ex(Ws, L, LI, s2, 32, [0.0, 1.0, float("inf"), 2.0], 2, codes, W, ws,
                              st) == E
    assert bk.bakron_round_ex(Ws, L, LI, s2, 32, list(range(32)), 5, codes, W, ws, st) == E
    assert bk.bakron_read_status(st) == 0
