"""Pins of the fp64 oracle against things other than itself (CPU only).

Each pin is chosen so that a plausible slip in the oracle (a dropped correction term, a
transposed factor, a wrong triangle, a wrong sign, the wrong rounding mode) fails it:

* U D U^T  vs numpy's Cholesky of the index-reversed matrix (a library routine);
* the rule vs GPTQ in its optimal-brain-surgeon form (a different algorithm) run on the
  vectorised problem with the explicit Kronecker Hessian H_O (x) H_I, and per row / per column
  when one factor is the identity;
* H_O = H_I = I vs plain round-to-nearest;
* brute-force enumeration of every code matrix: exactly one fixed point, equal to the oracle;
* the O(mn(m+n)) row sweep vs the raster definition;
* the loss identity tr(H_O E H_I E^T) = sum_ij D_O,i D_I,j Delta_ij^2 and the trace bound
  (YAQA article, section 4);
* invariance of the codes under H -> c H.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import (band_check, brute_force_fixed_points, code_range, fixed_point_pre,
                    fixed_point_pre_rows, gptq_obs, grid_quotient, proxy_loss, proxy_loss_kron,
                    quantize, round_naive, round_row_sweep, udu)
from two_sided_adaptive_bakron_b200.workloads import make_workload, random_problem


def _factors(HO, HI):
    LO, DO = udu(HO)
    LI, DI = udu(HI)
    return LO, DO, LI, DI


# ----------------------------------------------------------------------------- factorisation
@pytest.mark.parametrize("d,seed", [(1, 0), (2, 1), (7, 2), (40, 3), (129, 4)])
def test_udu_matches_reversed_cholesky(d, seed):
    _, H, _, _, _ = random_problem(d, 3, 2, seed)
    H = H.astype(np.float64)
    L, D = udu(H)
    assert np.all(np.tril(L) == 0.0)
    assert np.all(D > 0)
    P = np.eye(d)[::-1]
    C = np.linalg.cholesky(P @ H @ P)
    L_ref = P @ (C / np.diag(C)) @ P - np.eye(d)
    D_ref = (np.diag(C) ** 2)[::-1]
    np.testing.assert_allclose(L, L_ref, rtol=0, atol=1e-10 * max(1.0, np.abs(L_ref).max()))
    np.testing.assert_allclose(D, D_ref, rtol=1e-10)
    U = np.eye(d) + L
    rec = U @ np.diag(D) @ U.T
    assert np.abs(rec - H).max() <= 1e-12 * np.abs(H).max()


def test_udu_rejects_indefinite():
    H = np.array([[1.0, 2.0], [2.0, 1.0]])
    with pytest.raises(ValueError):
        udu(H)


# ----------------------------------------------------------------------------- base quantizer
def test_quantize_half_even_and_clamp():
    assert quantize(0.5, 1.0, 2) == 0
    assert quantize(1.5, 1.0, 4) == 2
    assert quantize(-0.5, 1.0, 2) == 0
    assert quantize(-2.5, 1.0, 4) == -2
    assert quantize(1.5, 1.0, 2) == 1     # rint -> 2, clamp to 1
    assert quantize(-9.7, 1.0, 4) == -8
    assert quantize(3.0, 0.0, 4) == 0     # zero scale row
    assert code_range(3) == (-4, 3)
    # the decision is on the real quotient: just below / above a half-integer (an fp32 quotient
    # would land on the tie and round to even instead)
    assert quantize(1.4999999999, 1.0, 4) == 1
    assert quantize(2.5000000001, 1.0, 4) == 3
    assert quantize(2.5, 1.0, 4) == 2 and quantize(3.5, 1.0, 4) == 4
    assert quantize(-7.5, 1.0, 4) == -8


def _exact_round(pre, s, bits):
    """Round half to even of the exact rational pre / s, then the clamp (Python fractions)."""
    lo, hi = code_range(bits)
    return min(max(round(Fraction(float(pre)) / Fraction(float(s))), lo), hi)


def test_quantize_equals_exact_rational_rounding_near_boundaries():
    # fp32 inputs placed on and within a few ulps of half-integer multiples of the grid step,
    # where a correctly rounded fp32 quotient would often fall on the tie itself
    rng = np.random.default_rng(17)
    hits = 0
    for _ in range(4000):
        s = np.float32(rng.uniform(1e-3, 1.0))
        k = int(rng.integers(-8, 8))
        pre = np.float32((k + 0.5) * float(s))
        pre = np.nextafter(pre, np.float32(np.inf) if rng.random() < 0.5 else np.float32(-np.inf)) \
            if rng.random() < 0.7 else pre
        exact = _exact_round(pre, s, 4)
        assert quantize(float(pre), float(s), 4) == exact, (pre, s)
        fp32q = np.float32(pre) / np.float32(s)
        hits += int(fp32q - np.floor(fp32q) == 0.5 and Fraction(float(pre)) / Fraction(float(s))
                    != Fraction(float(fp32q)))
    assert hits > 100   # the inputs do reach the cases where the fp32 quotient would mislead


# ----------------------------------------------------------------------------- special cases
@pytest.mark.parametrize("m,n,bits,seed", [(5, 9, 2, 0), (16, 33, 4, 1), (1, 17, 3, 2)])
def test_identity_factors_give_round_to_nearest(m, n, bits, seed):
    Ws, HO, HI, s, _ = random_problem(m, n, bits, seed, kind="identity")
    LO, _, LI, _ = _factors(HO, HI)
    C, _ = round_naive(Ws, LO, LI, s, bits)
    # round to nearest of the exact quotient (every row's largest entry sits near a tie)
    rtn = np.array([[_exact_round(Ws[i, j], s[i], bits) for j in range(n)] for i in range(m)])
    np.testing.assert_array_equal(C, rtn)


@pytest.mark.parametrize("m,n,bits,seed", [(4, 12, 2, 0), (3, 20, 3, 1), (6, 7, 4, 2)])
def test_ho_identity_is_rowwise_gptq(m, n, bits, seed):
    Ws, HO, HI, s, _ = random_problem(m, n, bits, seed, kind="ho_identity")
    LO, _, LI, _ = _factors(HO, HI)
    C, _ = round_naive(Ws, LO, LI, s, bits)
    for i in range(m):
        ref = gptq_obs(Ws[i], HI, np.full(n, s[i]), bits)
        np.testing.assert_array_equal(C[i], ref)


@pytest.mark.parametrize("m,n,bits,seed", [(12, 4, 2, 0), (20, 3, 3, 1)])
def test_hi_identity_is_columnwise_gptq(m, n, bits, seed):
    Ws, HO, HI, s, _ = random_problem(m, n, bits, seed, kind="hi_identity")
    LO, _, LI, _ = _factors(HO, HI)
    C, _ = round_naive(Ws, LO, LI, s, bits)
    for j in range(n):
        ref = gptq_obs(Ws[:, j], HO, s, bits)
        np.testing.assert_array_equal(C[:, j], ref)


@pytest.mark.parametrize("m,n,bits,seed", [(2, 4, 2, 0), (3, 4, 2, 1), (5, 7, 2, 2),
                                           (4, 6, 3, 3), (1, 6, 2, 4), (6, 1, 2, 5),
                                           (7, 5, 4, 6)])
def test_rule_is_gptq_on_vectorised_kronecker_problem(m, n, bits, seed):
    Ws, HO, HI, s, _ = random_problem(m, n, bits, seed)
    LO, _, LI, _ = _factors(HO, HI)
    C, _ = round_naive(Ws, LO, LI, s, bits)
    K = np.kron(HO.astype(np.float64), HI.astype(np.float64))
    ref = gptq_obs(Ws.reshape(-1), K, np.repeat(s, n), bits).reshape(m, n)
    np.testing.assert_array_equal(C, ref)


@pytest.mark.parametrize("m,n,seed", [(3, 3, 0), (2, 4, 1)])
def test_brute_force_unique_fixed_point(m, n, seed):
    Ws, HO, HI, s, bits = random_problem(m, n, 2, seed)
    LO, _, LI, _ = _factors(HO, HI)
    C, _ = round_naive(Ws, LO, LI, s, bits)
    found = brute_force_fixed_points(Ws, LO, LI, s, bits)
    assert len(found) == 1
    np.testing.assert_array_equal(found[0], C)


# ----------------------------------------------------------------------------- orders / forms
@pytest.mark.parametrize("name", ["small_64x128", "small_64x128_ho_identity",
                                  "small_64x128_identity"])
def test_row_sweep_equals_raster_definition(name):
    Ws, HO, HI, s, bits = make_workload(name)
    LO, _, LI, _ = _factors(HO, HI)
    C1, W1, P1 = round_naive(Ws, LO, LI, s, bits, return_pre=True)
    C2, W2, P2 = round_row_sweep(Ws, LO, LI, s, bits, return_pre=True)
    np.testing.assert_array_equal(C1, C2)
    np.testing.assert_allclose(P1, P2, rtol=0, atol=1e-12)


@pytest.mark.parametrize("m,n,bits,seed", [(13, 29, 2, 7), (31, 5, 3, 8), (1, 1, 2, 9)])
def test_row_sweep_equals_raster_ragged(m, n, bits, seed):
    Ws, HO, HI, s, _ = random_problem(m, n, bits, seed)
    LO, _, LI, _ = _factors(HO, HI)
    np.testing.assert_array_equal(round_naive(Ws, LO, LI, s, bits)[0],
                                  round_row_sweep(Ws, LO, LI, s, bits)[0])


def test_closed_form_fixed_point_holds():
    Ws, HO, HI, s, bits = make_workload("small_64x128")
    LO, _, LI, _ = _factors(HO, HI)
    C, W, P = round_naive(Ws, LO, LI, s, bits, return_pre=True)
    pre = fixed_point_pre(Ws, W, LO, LI)
    np.testing.assert_allclose(pre, P, rtol=0, atol=1e-12)
    lo, hi = code_range(bits)
    q = np.rint(grid_quotient(pre, np.broadcast_to(s[:, None], pre.shape)))
    np.testing.assert_array_equal(np.clip(q, lo, hi), C)


def test_zero_scale_row_gives_zero_codes():
    Ws, HO, HI, s, bits = random_problem(6, 10, 2, 3)
    Ws[2] = 0.0
    s = s.copy()
    s[2] = 0.0
    LO, _, LI, _ = _factors(HO, HI)
    C, W = round_naive(Ws, LO, LI, s, bits)
    assert np.all(C[2] == 0) and np.all(W[2] == 0)
    np.testing.assert_array_equal(C, round_row_sweep(Ws, LO, LI, s, bits)[0])


def test_codes_invariant_under_hessian_scaling():
    Ws, HO, HI, s, bits = make_workload("small_64x128")
    LO, _, LI, _ = _factors(HO, HI)
    LO2, _, LI2, _ = _factors(HO * np.float32(8.0), HI * np.float32(0.125))  # exact in fp32
    np.testing.assert_allclose(LO, LO2, atol=1e-12)
    np.testing.assert_array_equal(round_row_sweep(Ws, LO, LI, s, bits)[0],
                                  round_row_sweep(Ws, LO2, LI2, s, bits)[0])


# ----------------------------------------------------------------------------- loss
@pytest.mark.parametrize("m,n,seed", [(3, 4, 0), (5, 2, 1), (1, 6, 2)])
def test_proxy_loss_equals_explicit_kronecker_form(m, n, seed):
    rng = np.random.default_rng(seed)
    _, HO, HI, _, _ = random_problem(m, n, 2, seed)
    dW = rng.standard_normal((m, n))
    a = proxy_loss(dW, HO, HI)
    b = proxy_loss_kron(dW, HO, HI)
    assert abs(a - b) <= 1e-12 * abs(b)


@pytest.mark.parametrize("name", ["small_64x128", "small_64x128_ho_identity"])
def test_loss_identity_and_trace_bound(name):
    Ws, HO, HI, s, bits = make_workload(name)
    LO, DO, LI, DI = _factors(HO, HI)
    C, W, P = round_naive(Ws, LO, LI, s, bits, return_pre=True)
    E = Ws.astype(np.float64) - W
    delta = W - P
    loss = proxy_loss(E, HO, HI)
    ident = float(np.sum(DO[:, None] * DI[None, :] * delta ** 2))
    assert abs(loss - ident) <= 1e-9 * ident
    # YAQA article, section 4: dW (H_O (x) H_I) dW^T <= tr(D_I) tr(D_O) sigma^2
    sigma2 = float(np.max(delta ** 2))
    assert loss <= DO.sum() * DI.sum() * sigma2
    # unclamped entries have |Delta| <= s/2
    lo, hi = code_range(bits)
    inner = (C > lo) & (C < hi)
    assert np.all(np.abs(delta[inner]) <= 0.5 * s[:, None].repeat(C.shape[1], 1)[inner] + 1e-12)


# ----------------------------------------------------------------------------- the checkers
@pytest.mark.parametrize("m,n,seed", [(1, 1, 0), (13, 29, 1), (40, 7, 2), (64, 128, 3)])
def test_fixed_point_pre_rows_equals_full_closed_form(m, n, seed):
    # the row-restricted closed form (the checker of every large-shape test) against the full
    # one and against the raster definition's own pre values, for solved and arbitrary W
    Ws, HO, HI, s, bits = random_problem(m, n, 2, seed)
    LO, _, LI, _ = _factors(HO, HI)
    C, W, P = round_naive(Ws, LO, LI, s, bits, return_pre=True)
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, m - 1], rng.integers(0, m, 5)]))
    full = fixed_point_pre(Ws, W, LO, LI)
    got = fixed_point_pre_rows(Ws, W, LO, LI, rows)
    np.testing.assert_allclose(got, full[rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got, P[rows], rtol=0, atol=1e-12)
    shuffled = rows[::-1].copy()                      # any row order
    np.testing.assert_allclose(fixed_point_pre_rows(Ws, W, LO, LI, shuffled), full[shuffled],
                               rtol=0, atol=1e-12)
    Wr = rng.standard_normal((m, n))                  # the identity holds for any W
    np.testing.assert_allclose(fixed_point_pre_rows(Ws, Wr, LO, LI, rows),
                               fixed_point_pre(Ws, Wr, LO, LI)[rows], rtol=0, atol=1e-12)


def test_band_check_nearest_flags_wrong_codes():
    Ws, HO, HI, s, bits = make_workload("small_64x128")
    LO, _, LI, _ = _factors(HO, HI)
    C, W = round_naive(Ws, LO, LI, s, bits)
    pre = fixed_point_pre(Ws, W, LO, LI)
    assert band_check(pre, C, s, bits, 1e-3)[:2] == (0, 0)
    lo, hi = code_range(bits)
    # a code moved by one step, far from a boundary, is a mismatch outside the band
    x = pre / s[:, None]
    far = np.argwhere((np.abs(x - np.floor(x) - 0.5) > 0.1) & (C > lo) & (C < hi))
    i, j = far[len(far) // 2]
    Cb = C.copy()
    Cb[i, j] += 1
    assert band_check(pre, Cb, s, bits, 1e-3)[:2] == (1, 1)
    # the same move where pre/s sits 1e-4 steps from a half-integer is exempt (in the band)
    pre2 = pre.copy()
    pre2[i, j] = (np.floor(x[i, j]) + 0.5 + 1e-4) * s[i]
    Cc = C.copy()
    Cc[i, j] = np.floor(x[i, j])                     # nearest would be floor + 1
    mism, outside, in_band = band_check(pre2, Cc, s, bits, 1e-3)
    assert (mism, outside) == (1, 0) and in_band >= 1
    # and the band is what exempts it: with a narrower band the same entry is flagged
    assert band_check(pre2, Cc, s, bits, 1e-5)[:2] == (1, 1)
