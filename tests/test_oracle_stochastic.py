"""Pins of the oracle's stochastic Q (CPU only).

Stochastic rounding is the alternative to nearest rounding that the YAQA article's rounding
rule allows (section 4). The pins hold it to things other than itself:

* the from-definition Philox4x64-10 against numpy's Philox bit generator (a library routine
  of the same published generator);
* the variates: strictly inside (0, 1), on the 2^-16 midpoint grid, uniform;
* the base quantizer's defining property E[s floor(x + u)] = s x, over many seeds;
* a constant variate of 1/2 turns stochastic Q into nearest rounding (the pinned rule);
* with the identity as one factor, the rule with stochastic Q equals GPTQ (optimal brain
  surgeon form) run with the same variates; with both factors, GPTQ on the explicit
  Kronecker Hessian;
* brute force over every code matrix: exactly one fixed point of the closed form, equal to the
  oracle's; the row sweep and the raster definition agree entry by entry.
"""
import numpy as np
import pytest

from oracle import (band_check, brute_force_fixed_points, code_range, dither, fixed_point_pre,
                    gptq_obs, grid_quotient, philox4x64_10, quantize_stochastic,
                    round_naive, round_row_sweep, udu)
from two_sided_adaptive_bakron_b200.workloads import random_problem

M64 = (1 << 64) - 1


def _numpy_philox_block(counter, key):
    """numpy's Philox4x64-10 block at `counter`: its generator advances the counter before
    each block, so it is started one below (borrowing across the four words)."""
    words = [int(c) for c in counter]
    for w in range(4):
        if words[w] > 0:
            words[w] -= 1
            break
        words[w] = M64
    g = np.random.Philox(counter=np.array(words, dtype=np.uint64),
                         key=np.array([int(k) for k in key], dtype=np.uint64))
    return tuple(int(v) for v in g.random_raw(4))


@pytest.mark.parametrize("counter,key", [
    ((0, 0, 0, 0), (0, 0)),
    ((1, 0, 0, 0), (0, 0)),
    ((0, 5, 0, 0), (7, 0)),          # a borrow into word 1 on numpy's side
    ((3, 1000, 0, 0), (0xDEADBEEFCAFEF00D, 0)),
    ((M64, M64, M64, M64), (M64, M64)),
    ((0x243F6A8885A308D3, 0x13198A2E03707344, 0xA4093822299F31D0, 0x082EFA98EC4E6C89),
     (0x452821E638D01377, 0xBE5466CF34E90C6C)),
])
def test_philox_matches_numpy(counter, key):
    assert philox4x64_10(counter, key) == _numpy_philox_block(counter, key)


def test_dither_fields_and_distribution():
    m, n, seed = 37, 300, 11
    U = dither(m, n, seed)
    assert U.shape == (m, n)
    assert np.all(U > 0) and np.all(U < 1)
    k = U * 65536.0 - 0.5                      # the 16-bit fields
    assert np.all(k == np.round(k)) and k.min() >= 0 and k.max() <= 65535
    # the field of (i, j): block (j // 16, i), word (j % 16) // 4, bits 16 (j % 4)
    i, j = 23, 181
    w = philox4x64_10((j // 16, i, 0, 0), (seed, 0))
    assert k[i, j] == (w[(j % 16) // 4] >> (16 * (j % 4))) & 0xFFFF
    # a row subset gives the same rows
    np.testing.assert_array_equal(dither([5, 30], n, seed), U[[5, 30]])
    # uniform: mean 1/2 and variance 1/12 within a few standard errors, flat deciles
    N = U.size
    assert abs(U.mean() - 0.5) < 5 * np.sqrt(1 / 12 / N)
    assert abs(U.var() - 1 / 12) < 5 * np.sqrt(1 / 180 / N)
    counts = np.histogram(U, bins=10, range=(0, 1))[0]
    chi2 = ((counts - N / 10) ** 2 / (N / 10)).sum()
    assert chi2 < 40                            # 9 degrees of freedom
    # another seed gives other variates
    assert np.mean(dither(m, n, seed + 1) == U) < 0.01


def test_quantize_stochastic_cases():
    # x = 0.25: up iff u >= 0.75
    assert quantize_stochastic(0.25, 1.0, 4, 0.7) == 0
    assert quantize_stochastic(0.25, 1.0, 4, 0.8) == 1
    # negative x = -1.25: floor(-1.25 + u) is -2 for u < 0.25, -1 above
    assert quantize_stochastic(-1.25, 1.0, 4, 0.2) == -2
    assert quantize_stochastic(-1.25, 1.0, 4, 0.3) == -1
    # clamp and the zero-scale row
    assert quantize_stochastic(7.6, 1.0, 4, 0.5) == 7
    assert quantize_stochastic(-8.9, 1.0, 4, 0.05) == -8
    assert quantize_stochastic(3.0, 0.0, 4, 0.5) == 0
    # integers stay put for any u < 1
    assert quantize_stochastic(2.0, 0.5, 4, 0.99998) == 4
    # the sum is the real one: 0.49999997 (fp32) + 0.5 stays below 1 (an fp32 addition would
    # round it up to 1.0)
    x = float(np.float32(0.5) - np.float32(2.0 ** -25))
    assert quantize_stochastic(x, 1.0, 4, 0.5) == 0
    assert quantize_stochastic(0.5, 1.0, 4, 0.5) == 1


def test_stochastic_q_is_unbiased():
    # the identity factors reduce the rule to Q itself: E[W] = W* away from the clamp
    m, n, bits = 24, 40, 4
    Ws, _, _, s, _ = random_problem(m, n, bits, 5, kind="identity")
    LO, LI = np.zeros((m, m)), np.zeros((n, n))
    seeds = 300
    acc = np.zeros((m, n))
    for sd in range(seeds):
        C, W = round_naive(Ws, LO, LI, s, bits, dither=dither(m, n, sd))
        fl = np.floor(Ws.astype(np.float64) / s[:, None])
        assert np.all((C == fl) | (C == fl + 1) | (C == code_range(bits)[1]))
        acc += W
    x = Ws.astype(np.float64) / s[:, None]
    ok = np.abs(x) < 6.9                        # no clamping possible
    err = (acc / seeds - Ws)[ok] / np.broadcast_to(s[:, None], (m, n))[ok]
    assert np.abs(err).max() < 6 * 0.5 / np.sqrt(seeds)
    assert abs(err.mean()) < 5 * 0.5 / np.sqrt(seeds * err.size)
    # the dither matters: nearest rounding has a systematic bias on the same entries
    C0, W0 = round_naive(Ws, LO, LI, s, bits)
    assert np.abs((W0 - Ws)[ok]).mean() > 5 * np.abs((acc / seeds - Ws)[ok]).mean()


@pytest.mark.parametrize("kind", ["identity", "kron"])
def test_half_dither_is_nearest(kind):
    # floor(x + 1/2) is nearest rounding except at exact ties, where it rounds up instead of to
    # even. With identity factors pre = W*; power-of-two grid steps and entries placed on
    # half-integer multiples of them make exact ties.
    m, n, bits = 12, 20, 3
    Ws, HO, HI, s, _ = random_problem(m, n, bits, 2, kind=kind)
    if kind == "identity":
        rng = np.random.default_rng(3)
        s = (2.0 ** -(3 + np.arange(m) % 3)).astype(np.float32)
        Ws = Ws.copy()
        for i in range(m):
            cols = rng.choice(n, 4, replace=False)
            Ws[i, cols] = (rng.integers(-4, 3, 4) + 0.5) * s[i]
    LO, _ = udu(HO)
    LI, _ = udu(HI)
    C0, W0, P0 = round_naive(Ws, LO, LI, s, bits, return_pre=True)
    C1, W1 = round_naive(Ws, LO, LI, s, bits, dither=np.full((m, n), 0.5))
    xq = grid_quotient(P0, np.broadcast_to(s[:, None], P0.shape))
    tie = xq - np.floor(xq) == 0.5
    if kind == "identity":
        assert tie.sum() == 4 * m
        np.testing.assert_array_equal(C1[tie], np.minimum(np.floor(xq[tie]) + 1, code_range(bits)[1]))
        assert np.all(C0[tie] % 2 == 0)
    else:
        assert tie.sum() == 0
    np.testing.assert_array_equal(C0[~tie], C1[~tie])
    np.testing.assert_array_equal(W0[~tie], W1[~tie])


@pytest.mark.parametrize("side", ["in", "out"])
def test_one_sided_stochastic_matches_gptq(side):
    m, n, bits = 6, 14, 3
    Ws, HO, HI, s, _ = random_problem(m, n, bits, 7)
    U = dither(m, n, 99)
    if side == "in":          # H_O = I: every row is GPTQ under H_I
        LO, LI = np.zeros((m, m)), udu(HI)[0]
        C, _ = round_naive(Ws, LO, LI, s, bits, dither=U)
        for i in range(m):
            ref = gptq_obs(Ws[i], HI, np.full(n, s[i]), bits, dither=U[i])
            np.testing.assert_array_equal(C[i], ref)
    else:                     # H_I = I: every column is GPTQ under H_O
        LO, LI = udu(HO)[0], np.zeros((n, n))
        C, _ = round_naive(Ws, LO, LI, s, bits, dither=U)
        for j in range(n):
            ref = gptq_obs(Ws[:, j], HO, s, bits, dither=U[:, j])
            np.testing.assert_array_equal(C[:, j], ref)


def test_two_sided_stochastic_matches_gptq_on_kron():
    m, n, bits = 4, 6, 2
    Ws, HO, HI, s, _ = random_problem(m, n, bits, 8)
    U = dither(m, n, 3)
    LO, LI = udu(HO)[0], udu(HI)[0]
    C, _ = round_naive(Ws, LO, LI, s, bits, dither=U)
    K = np.kron(HO.astype(np.float64), HI.astype(np.float64))
    ref = gptq_obs(Ws.reshape(-1), K, np.repeat(s, n), bits, dither=U.reshape(-1))
    np.testing.assert_array_equal(C, ref.reshape(m, n))


@pytest.mark.parametrize("m,n,seed", [(3, 3, 0), (2, 4, 1)])
def test_stochastic_brute_force_unique_fixed_point(m, n, seed):
    bits = 2
    Ws, HO, HI, s, _ = random_problem(m, n, bits, seed + 20)
    LO, LI = udu(HO)[0], udu(HI)[0]
    U = dither(m, n, seed)
    found = brute_force_fixed_points(Ws, LO, LI, s, bits, dither=U)
    assert len(found) == 1
    C, _ = round_naive(Ws, LO, LI, s, bits, dither=U)
    np.testing.assert_array_equal(found[0], C)


@pytest.mark.parametrize("m,n,bits,seed", [(9, 13, 2, 0), (17, 11, 4, 1)])
def test_stochastic_row_sweep_and_closed_form(m, n, bits, seed):
    Ws, HO, HI, s, _ = random_problem(m, n, bits, seed + 30)
    LO, LI = udu(HO)[0], udu(HI)[0]
    U = dither(m, n, 1234 + seed)
    C, W, P = round_naive(Ws, LO, LI, s, bits, return_pre=True, dither=U)
    C2, W2 = round_row_sweep(Ws, LO, LI, s, bits, dither=U)
    np.testing.assert_array_equal(C, C2)
    pre = fixed_point_pre(Ws, W, LO, LI)
    np.testing.assert_allclose(pre, P, rtol=0, atol=1e-12 * max(1.0, np.abs(P).max()))
    mism, outside, _ = band_check(pre, C, s, bits, 1e-9, dither=U)
    assert mism == 0 and outside == 0
    # band_check sees a wrong code
    Cb = C.copy()
    Cb[m // 2, n // 2] += 1 if Cb[m // 2, n // 2] < code_range(bits)[1] else -1
    assert band_check(pre, Cb, s, bits, 1e-9, dither=U)[1] == 1
    # stochastic codes differ from nearest on a good share of the entries
    C0, _ = round_naive(Ws, LO, LI, s, bits)
    assert np.mean(C0 != C) > 0.1
    # the grid decision is floor(pre / s + u) on the real values
    i, j = 1, 2
    assert C[i, j] == np.clip(np.floor(P[i, j] / s[i] + U[i, j]), *code_range(bits))
