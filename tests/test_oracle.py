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
import numpy as np
import pytest

from oracle import (brute_force_fixed_points, code_range, fixed_point_pre, gptq_obs, grid_quotient,
                    proxy_loss, proxy_loss_kron, quantize, round_naive, round_row_sweep, udu)
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
    # the decision is taken on the fp32 quotient: 0.7499999999 rounds to fp32 0.75 -> 1
    assert quantize(0.7499999999, 1.0, 4) == 1
    assert quantize(-7.5, 1.0, 4) == -8


# ----------------------------------------------------------------------------- special cases
@pytest.mark.parametrize("m,n,bits,seed", [(5, 9, 2, 0), (16, 33, 4, 1), (1, 17, 3, 2)])
def test_identity_factors_give_round_to_nearest(m, n, bits, seed):
    Ws, HO, HI, s, _ = random_problem(m, n, bits, seed, kind="identity")
    LO, _, LI, _ = _factors(HO, HI)
    C, _ = round_naive(Ws, LO, LI, s, bits)
    lo, hi = code_range(bits)
    # round to nearest, the quotient taken as one fp32 division (the decision precision)
    rtn = np.clip(np.rint(Ws.astype(np.float32) / s[:, None].astype(np.float32)), lo, hi)
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
