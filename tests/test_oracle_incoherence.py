"""Pins of the oracle's incoherence processing (CPU only): the randomised Hadamard transform
T_d = H_d S_d / sqrt(d) on both sides of the layer and of the Kronecker factors (YAQA article,
section 4: lower the factors' incoherence before quantising, as LDLQ does).

* Sylvester's H_{2^k} against scipy.linalg.hadamard (a library routine);
* the GF(27) arithmetic behind Paley's H_28: every nonzero element has an inverse, the
  quadratic character is multiplicative with chi(-1) = -1 (27 = 3 mod 4);
* H_28 and H_28 (x) H_{2^k}: +-1 entries, H H^T = d I, H_28 skew (H + H^T = 2 I);
* the signs: +-1, balanced, seed-dependent, each the stated bit of its Philox block;
* T orthogonal, the inverse undoes the forward transform, norms are kept, a spike becomes
  flat, and the proxy loss tr(H_O dW H_I dW^T) is the same in the rotated basis.
"""
import numpy as np
import pytest
import scipy.linalg

from oracle import (gf27_chi, hadamard, hadamard28, hadamard_rows, philox4x64_10, proxy_loss, rht,
                    rht_matrix, rht_signs)
from oracle.bakron_oracle import _gf27, _gf27_mul


@pytest.mark.parametrize("k", [1, 2, 4, 8, 64, 512])
def test_sylvester_matches_scipy(k):
    np.testing.assert_array_equal(hadamard(k), scipy.linalg.hadamard(k))


def test_gf27_field_and_character():
    one = (1, 0, 0)
    elems = [_gf27(e) for e in range(27)]
    for a in elems[1:]:
        assert sum(_gf27_mul(a, b) == one for b in elems[1:]) == 1      # a unique inverse
    chi = gf27_chi()
    index = {el: e for e, el in enumerate(elems)}
    for a in range(1, 27):
        for b in range(1, 27):
            assert chi[index[_gf27_mul(elems[a], elems[b])]] == chi[a] * chi[b]
    minus_one = index[(2, 0, 0)]
    assert chi[minus_one] == -1
    assert chi[0] == 0 and (chi == 1).sum() == 13


@pytest.mark.parametrize("d", [28, 56, 112, 448])
def test_hadamard_orthogonal(d):
    H = hadamard(d)
    assert set(np.unique(H)) == {-1.0, 1.0}
    np.testing.assert_array_equal(H @ H.T, d * np.eye(d))
    H28 = hadamard28()
    np.testing.assert_array_equal(H28 + H28.T, 2 * np.eye(28))


@pytest.mark.parametrize("d", [3, 12, 20, 84])
def test_unsupported_sizes_raise(d):
    with pytest.raises(ValueError):
        hadamard(d)


def test_signs():
    s = rht_signs(1 << 14, 9)
    assert set(np.unique(s)) == {-1.0, 1.0}
    assert abs(s.mean()) < 5 / np.sqrt(s.size)
    assert np.mean(rht_signs(1 << 14, 10) == s) < 0.6
    i = 1000
    w = philox4x64_10((i // 256, 0, 1, 0), (9, 0))
    bit = (w[(i % 256) // 64] >> (i % 64)) & 1
    assert s[i] == (-1.0 if bit else 1.0)


@pytest.mark.parametrize("r,c", [(8, 28), (56, 16), (32, 112)])
def test_rht_orthogonal_and_invertible(r, c):
    rng = np.random.default_rng(r + c)
    for d in (r, c):
        T = rht_matrix(d, 3)
        np.testing.assert_allclose(T @ T.T, np.eye(d), atol=1e-13)
    X = rng.standard_normal((r, c))
    Y = rht(X, 3, 4)
    np.testing.assert_allclose(rht(Y, 3, 4, inverse=True), X, atol=1e-12)
    assert abs(np.linalg.norm(Y) - np.linalg.norm(X)) < 1e-12 * np.linalg.norm(X)
    spike = np.zeros((r, c))
    spike[r // 3, c // 2] = 1.0
    np.testing.assert_allclose(np.abs(rht(spike, 3, 4)), 1.0 / np.sqrt(r * c), rtol=1e-12)


def test_proxy_loss_is_invariant():
    rng = np.random.default_rng(7)
    m, n = 16, 56
    dW = rng.standard_normal((m, n))
    A, B = rng.standard_normal((m, m)), rng.standard_normal((n, n))
    HO, HI = A @ A.T + np.eye(m), B @ B.T + np.eye(n)
    so, si = 21, 22
    dWt, HOt, HIt = rht(dW, so, si), rht(HO, so, so), rht(HI, si, si)
    assert abs(proxy_loss(dWt, HOt, HIt) - proxy_loss(dW, HO, HI)) < 1e-10 * proxy_loss(dW, HO, HI)


@pytest.mark.parametrize("d", [1, 8, 28, 112])
def test_hadamard_rows_are_rows_of_hadamard(d):
    rows = np.array([0, d - 1, d // 2, d // 3])
    np.testing.assert_array_equal(hadamard_rows(d, rows), hadamard(d)[rows])
