"""The solver's acceptance gate at full size, through the path the benchmark times (B200).

For every layer workload (64x128 with its two variants, 1024^2, 4096^2, 4096x14336 and
28672x8192), the whole path runs on the device exactly as ``bench.py`` launches it
(``Solver.run``: bakron_ldl of H_O on a side stream and of H_I on the caller's stream, then
bakron_round with the library's own factors, then bakron_proxy_loss), and the host checks in
fp64 with the oracle:

* the rounding rule (YAQA article, section 4) through its closed form: at EVERY entry,
  code = Q(W* + (I + L_O)^T E (I + L_I) - E) with the factors the library produced, except
  where pre/s lies within 1e-3 grid steps of a rounding boundary, and such exempt mismatches
  are at most 0.1% of the entries (evaluated by row blocks with ``oracle.fixed_point_pre_rows``
  and ``oracle.band_check``);
* the proxy loss tr(H_O dW H_I dW^T) within 1e-3 relative of ``oracle.proxy_loss``;
* both factorisations H = (I + L) D (I + L)^T (same section): L strictly upper, D > 0, the
  backward error on sampled rows within 4 d eps_32 of |I + L| D |I + L|^T, and the forward
  error against a library Cholesky of the reversed matrix (fp64) within 50 kappa eps_32.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import band_check, code_range, fixed_point_pre_rows, proxy_loss
from two_sided_adaptive_bakron_b200.workloads import WORKLOADS, make_workload

from ._helpers import cond_estimate, library_udu, library_udu_torch, udu_backward_error_rows

pytestmark = pytest.mark.gpu

BAND = 1e-3
MAX_EXEMPT_FRAC = 1e-3
EPS32 = 2.0 ** -24


@pytest.fixture(scope="module")
def bk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from two_sided_adaptive_bakron_b200 import build
    build.build()
    from two_sided_adaptive_bakron_b200 import bakron
    return bakron


def _check_factor(H, L, D, name):
    d = H.shape[0]
    Ld = torch.from_numpy(L).cuda()
    assert bool(torch.all(torch.tril(Ld) == 0)), f"{name}: L not strictly upper"
    del Ld
    assert np.all(np.isfinite(D)) and np.all(D > 0), f"{name}: pivots"
    rng = np.random.default_rng(d)
    rows = np.unique(np.concatenate([[0, 1, d // 2, d - 2, d - 1], rng.integers(0, d, 27)]))
    rows = rows[(rows >= 0) & (rows < d)]
    err, scale = udu_backward_error_rows(H, L, D, rows)
    assert err <= 4 * d * EPS32 * scale, (name, err, scale)
    L_ref, D_ref = library_udu(H) if d <= 2048 else library_udu_torch(H, "cuda")
    kappa = cond_estimate(H, "cuda")
    tol = 50 * kappa * EPS32
    fwd = float(np.abs(L.astype(np.float64) - L_ref).max()) / max(1.0, float(np.abs(L_ref).max()))
    assert fwd <= tol, (name, fwd, kappa)
    drel = float(np.max(np.abs(D.astype(np.float64) - D_ref) / D_ref))
    assert drel <= tol, (name, drel, kappa)


@pytest.mark.parametrize("name", ["small_64x128", "small_64x128_ho_identity",
                                  "small_64x128_identity", "sq_1024", "attn_4096",
                                  "down_4096x14336", "upgate_28672x8192"])
def test_whole_path_full_size(bk, name):
    wl = WORKLOADS[name]
    Ws, HO, HI, s, bits = make_workload(wl, device="cuda" if wl.m * wl.n > (1 << 22) else None)
    m, n = Ws.shape
    solver = bk.Solver(m, n, "cuda")
    d = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    dWs, dHO, dHI, ds = d(Ws), d(HO), d(HI), d(s)
    solver.run(dWs, dHO, dHI, ds, bits)
    solver.check()
    torch.cuda.synchronize()
    C = solver.codes.cpu().numpy()
    W = solver.W.cpu().numpy()
    LO, DO = solver.L_O.cpu().numpy(), solver.D_O.cpu().numpy()
    LI, DI = solver.L_I.cpu().numpy(), solver.D_I.cpu().numpy()
    loss = float(solver.loss.item())
    del solver, dWs, dHO, dHI, ds
    torch.cuda.empty_cache()

    lo, hi = code_range(bits)
    assert C.min() >= lo and C.max() <= hi
    np.testing.assert_array_equal(W, (s[:, None] * C.astype(np.float32)).astype(np.float32))

    # the rule at every entry, with the library's own factors
    Ws64, W64, LI64 = Ws.astype(np.float64), W.astype(np.float64), LI.astype(np.float64)
    mism = outside = in_band = 0
    chunk = max(1, min(m, (1 << 24) // n))
    for r0 in range(0, m, chunk):
        rows = np.arange(r0, min(m, r0 + chunk))
        pre = fixed_point_pre_rows(Ws64, W64, LO, LI64, rows)
        a, b, c = band_check(pre, C[rows], s[rows], bits, BAND)
        mism, outside, in_band = mism + a, outside + b, in_band + c
    assert outside == 0, (name, mism, outside, in_band)
    assert mism <= MAX_EXEMPT_FRAC * m * n, (name, mism, in_band)
    del LI64

    # the loss of the residual the round left behind
    ref = proxy_loss(Ws64 - W64, HO, HI)
    assert abs(loss - ref) <= 1e-3 * abs(ref), (name, loss, ref)
    del Ws64, W64

    # both factorisations
    _check_factor(HO, LO, DO, name + ":H_O")
    _check_factor(HI, LI, DI, name + ":H_I")
