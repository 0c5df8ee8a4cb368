"""Pins of the oracle's pluggable base quantizer (CPU only): per-group grid steps and sorted
scalar codebooks (the BaKron page's summary: the solver is modular in the base quantizer).

* a codebook decision against the argmin over entries (a different formula from the midpoint
  count), ties to the lower entry, the ends of the range, a zero-scale row;
* the codebook of the integers is the uniform quantizer (away from exact ties);
* one group of n columns is the per-row scale; with identity factors the rule is plain
  round-to-nearest per group / per codebook;
* with one factor the identity, GPTQ (optimal brain surgeon form) with the same quantizer, per
  row and per column; with both, GPTQ on the explicit Kronecker Hessian;
* brute force: exactly one fixed point, equal to the oracle's; row sweep = raster definition;
  the closed-form fixed point holds entry by entry.
"""
import numpy as np
import pytest

from oracle import (band_check, brute_force_fixed_points, code_range, codebook_midpoints,
                    fixed_point_pre, gptq_obs, grid_quotient, quantize_codebook, round_naive,
                    round_row_sweep, udu)
from two_sided_adaptive_bakron_b200.workloads import random_problem

CB3 = np.array([-1.0, -0.62, -0.33, -0.1, 0.08, 0.3, 0.61, 1.0], dtype=np.float32)


def _group_scales(Ws, gs, top):
    m, n = Ws.shape
    G = (n + gs - 1) // gs
    s = np.zeros((m, G), dtype=np.float32)
    for g in range(G):
        s[:, g] = np.abs(Ws[:, g * gs:(g + 1) * gs]).max(axis=1) / np.float32(top)
    return s


def test_codebook_decision_cases():
    cb = np.array([-1.0, -0.25, 0.5, 2.0], dtype=np.float32)
    mids = codebook_midpoints(cb)
    np.testing.assert_array_equal(mids, [-0.625, 0.125, 1.25])
    for x in (-3.0, -0.7, -0.6, 0.0, 0.124, 0.126, 1.0, 1.3, 9.0):
        ref = int(np.argmin(np.abs(cb.astype(np.float64) - x)))
        assert quantize_codebook(x, 1.0, cb) == ref, x
    assert quantize_codebook(0.125, 1.0, cb) == 1       # a tie goes to the lower entry
    assert quantize_codebook(-0.625, 1.0, cb) == 0
    assert quantize_codebook(5.0, 0.0, cb) == 0         # zero-scale row
    assert quantize_codebook(0.75, 0.5, cb) == 3        # x = 1.5


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_integer_codebook_is_the_uniform_quantizer(bits):
    m, n = 9, 14
    Ws, HO, HI, s, _ = random_problem(m, n, bits, 40 + bits)
    LO, LI = udu(HO)[0], udu(HI)[0]
    lo, hi = code_range(bits)
    C0, W0, P0 = round_naive(Ws, LO, LI, s, bits, return_pre=True)
    C1, W1 = round_naive(Ws, LO, LI, s, bits, codebook=np.arange(lo, hi + 1, dtype=np.float32))
    xq = grid_quotient(P0, np.broadcast_to(s[:, None], P0.shape))
    assert not np.any(xq - np.floor(xq) == 0.5)         # no exact ties on this input
    np.testing.assert_array_equal(C1 + lo, C0)
    np.testing.assert_allclose(W1, W0, rtol=1e-7)


def test_one_group_is_per_row():
    m, n, bits = 7, 20, 3
    Ws, HO, HI, s, _ = random_problem(m, n, bits, 5)
    LO, LI = udu(HO)[0], udu(HI)[0]
    C0, W0 = round_naive(Ws, LO, LI, s, bits)
    C1, W1 = round_naive(Ws, LO, LI, s[:, None], bits, group_size=n)
    np.testing.assert_array_equal(C0, C1)
    np.testing.assert_array_equal(W0, W1)


def test_identity_factors_round_to_nearest_per_group_and_codebook():
    m, n, bits, gs = 6, 40, 4, 16
    Ws, _, _, _, _ = random_problem(m, n, bits, 6, kind="identity")
    sg = _group_scales(Ws, gs, 7.5)
    Z_O, Z_I = np.zeros((m, m)), np.zeros((n, n))
    C, _ = round_naive(Ws, Z_O, Z_I, sg, bits, group_size=gs)
    lo, hi = code_range(bits)
    sfull = np.repeat(sg, gs, axis=1)[:, :n]
    np.testing.assert_array_equal(
        C, np.clip(np.rint(Ws.astype(np.float64) / sfull.astype(np.float64)), lo, hi))
    sc = _group_scales(Ws, gs, 1.0)
    C, W = round_naive(Ws, Z_O, Z_I, sc, 3, codebook=CB3, group_size=gs)
    sfull = np.repeat(sc, gs, axis=1)[:, :n].astype(np.float64)
    ref = np.argmin(np.abs(CB3.astype(np.float64)[None, None, :] - (Ws / sfull)[..., None]),
                    axis=-1)
    np.testing.assert_array_equal(C, ref)
    np.testing.assert_allclose(W, sfull * CB3[C], rtol=1e-7)


@pytest.mark.parametrize("side", ["in", "out"])
def test_one_sided_codebook_matches_gptq(side):
    m, n = 5, 12
    Ws, HO, HI, _, _ = random_problem(m, n, 3, 8)
    s = (np.abs(Ws).max(axis=1) / np.float32(1.0)).astype(np.float32)
    if side == "in":
        LO, LI = np.zeros((m, m)), udu(HI)[0]
        C, _ = round_naive(Ws, LO, LI, s, 3, codebook=CB3)
        for i in range(m):
            np.testing.assert_array_equal(C[i], gptq_obs(Ws[i], HI, np.full(n, s[i]), 3,
                                                         codebook=CB3))
    else:
        LO, LI = udu(HO)[0], np.zeros((n, n))
        C, _ = round_naive(Ws, LO, LI, s, 3, codebook=CB3)
        for j in range(n):
            np.testing.assert_array_equal(C[:, j], gptq_obs(Ws[:, j], HO, s, 3, codebook=CB3))


def test_two_sided_groups_and_codebook_match_gptq_on_kron():
    m, n, gs = 4, 6, 3
    Ws, HO, HI, _, _ = random_problem(m, n, 3, 9)
    sg = _group_scales(Ws, gs, 1.0)
    LO, LI = udu(HO)[0], udu(HI)[0]
    C, _ = round_naive(Ws, LO, LI, sg, 3, codebook=CB3, group_size=gs)
    K = np.kron(HO.astype(np.float64), HI.astype(np.float64))
    per_coord = np.repeat(sg, gs, axis=1)[:, :n].reshape(-1)
    ref = gptq_obs(Ws.reshape(-1), K, per_coord, 3, codebook=CB3).reshape(m, n)
    np.testing.assert_array_equal(C, ref)


@pytest.mark.parametrize("m,n,seed", [(3, 3, 0), (2, 4, 1)])
def test_codebook_brute_force_unique_fixed_point(m, n, seed):
    cb = np.array([-1.0, -0.2, 0.35, 1.0], dtype=np.float32)
    Ws, HO, HI, _, _ = random_problem(m, n, 2, seed + 50)
    s = (np.abs(Ws).max(axis=1)).astype(np.float32)
    LO, LI = udu(HO)[0], udu(HI)[0]
    found = brute_force_fixed_points(Ws, LO, LI, s, 2, codebook=cb)
    assert len(found) == 1
    C, _ = round_naive(Ws, LO, LI, s, 2, codebook=cb)
    np.testing.assert_array_equal(found[0], C)


@pytest.mark.parametrize("m,n,gs,use_cb,seed", [(9, 40, 8, False, 0), (13, 37, 16, True, 1),
                                                (6, 64, 32, True, 2)])
def test_groups_codebook_row_sweep_and_closed_form(m, n, gs, use_cb, seed):
    bits = 3
    Ws, HO, HI, _, _ = random_problem(m, n, bits, seed + 60)
    cb = CB3 if use_cb else None
    sg = _group_scales(Ws, gs, 1.0 if use_cb else 3.5)
    LO, LI = udu(HO)[0], udu(HI)[0]
    C, W, P = round_naive(Ws, LO, LI, sg, bits, return_pre=True, codebook=cb, group_size=gs)
    C2, W2 = round_row_sweep(Ws, LO, LI, sg, bits, codebook=cb, group_size=gs)
    np.testing.assert_array_equal(C, C2)
    pre = fixed_point_pre(Ws, W, LO, LI)
    np.testing.assert_allclose(pre, P, rtol=0, atol=1e-12 * max(1.0, np.abs(P).max()))
    mism, outside, _ = band_check(pre, C, sg, bits, 1e-9, codebook=cb, group_size=gs)
    assert mism == 0 and outside == 0
    Cb = C.copy()
    Cb[m // 2, n // 2] = (Cb[m // 2, n // 2] + 1) % (len(CB3) if use_cb else 2)
    assert band_check(pre, Cb, sg, bits, 1e-9, codebook=cb, group_size=gs)[1] >= 1
