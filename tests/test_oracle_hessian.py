"""Pins of the oracle's Kronecker-factor construction (CPU only).

The YAQA article, section 3, builds the factors as second moments: H_1 = E[x^T x] over input
rows, and Sketch B, one power-iteration round from the identity, H_I = E_s[G_s^T G_s] / m,
H_O = E_s[G_s G_s^T] / n over per-sequence gradients G_s. The pins hold the oracle to things
other than itself:

* the Gram by explicit sums over samples on tiny inputs (no matrix product);
* closed forms: the trace identity tr(X^T X / N) = |X|_F^2 / N, orthonormal columns giving the
  identity, identical rows giving a rank-one v v^T, scaling by c giving c^2;
* Sketch B against the explicit Fisher E_s[vec(G_s) vec(G_s)^T] (mn x mn, row-major vec) and
  its two partial traces, which is what one power-iteration step from the identity computes;
* the damping adds damp * mean(diag) to the diagonal only;
* Sketch A: no round is the one-sided start, one round written out token by token, tokens
  that all share one x and one g keep x^T x and g^T g as the factors' shapes, and the
  c^2 scaling of both factors when the gradients scale by c.
"""
import numpy as np
import pytest

from oracle import damped_gram, damped_gram_rows, sketch_a, sketch_b


def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("N,d,seed", [(1, 1, 0), (3, 4, 1), (9, 5, 2)])
def test_gram_by_explicit_sums(N, d, seed):
    X = _rng(seed).standard_normal((N, d))
    damp = 0.01
    G = np.zeros((d, d))
    for a in range(d):
        for b in range(d):
            acc = 0.0
            for t in range(N):
                acc += X[t, a] * X[t, b]
            G[a, b] = acc / N
    mean_diag = sum(G[a, a] for a in range(d)) / d
    for a in range(d):
        G[a, a] += damp * mean_diag
    np.testing.assert_allclose(damped_gram(X, damp), G, rtol=1e-13, atol=1e-15)


def test_gram_closed_forms():
    rng = _rng(3)
    N, d = 50, 12
    X = rng.standard_normal((N, d))
    H = damped_gram(X, 0.0)
    assert abs(np.trace(H) - (X ** 2).sum() / N) < 1e-12 * np.trace(H)
    np.testing.assert_array_equal(H, H.T)
    assert np.linalg.eigvalsh(H).min() > -1e-12
    # orthonormal columns scaled by sqrt(N): the identity, then (1 + damp) I
    Q, _ = np.linalg.qr(rng.standard_normal((N, d)))
    np.testing.assert_allclose(damped_gram(np.sqrt(N) * Q, 0.0), np.eye(d), atol=1e-12)
    np.testing.assert_allclose(damped_gram(np.sqrt(N) * Q, 0.25), 1.25 * np.eye(d), atol=1e-12)
    # identical rows v: v v^T
    v = rng.standard_normal(d)
    np.testing.assert_allclose(damped_gram(np.tile(v, (7, 1)), 0.0), np.outer(v, v), atol=1e-12)
    # scaling and row order
    np.testing.assert_allclose(damped_gram(3.0 * X, 0.01), 9.0 * damped_gram(X, 0.01), rtol=1e-12)
    np.testing.assert_allclose(damped_gram(X[::-1], 0.01), damped_gram(X, 0.01), rtol=1e-12)


def test_damping_on_the_diagonal_only():
    X = _rng(4).standard_normal((30, 6))
    H0, H1 = damped_gram(X, 0.0), damped_gram(X, 0.1)
    off = ~np.eye(6, dtype=bool)
    np.testing.assert_array_equal(H0[off], H1[off])
    np.testing.assert_allclose(np.diag(H1) - np.diag(H0), 0.1 * np.mean(np.diag(H0)), rtol=1e-12)
    # the damped factor is positive definite even for a rank-deficient X
    Xr = np.tile(X[:1], (5, 1))
    assert np.linalg.eigvalsh(damped_gram(Xr, 0.01)).min() > 0


@pytest.mark.parametrize("S,m,n,seed", [(1, 2, 3, 0), (4, 3, 5, 1), (7, 5, 4, 2)])
def test_sketch_b_is_partial_trace_of_fisher(S, m, n, seed):
    G = _rng(seed).standard_normal((S, m, n))
    damp = 0.02
    # the Fisher of the vectorised weights (row-major vec: index a n + j)
    F = sum(np.outer(G[s].reshape(-1), G[s].reshape(-1)) for s in range(S)) / S
    F4 = F.reshape(m, n, m, n)                       # F4[a, j, b, l]
    HI_ref = np.einsum("ajal->jl", F4) / m            # one step from H_O = I: tr over outputs
    HO_ref = np.einsum("ajbj->ab", F4) / n            # one step from H_I = I: tr over inputs
    HI_ref[np.diag_indices(n)] += damp * np.trace(HI_ref) / n
    HO_ref[np.diag_indices(m)] += damp * np.trace(HO_ref) / m
    HO, HI = sketch_b(G, damp)
    np.testing.assert_allclose(HI, HI_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(HO, HO_ref, rtol=1e-12, atol=1e-14)
    # the same factors as Grams of the stacked gradients
    np.testing.assert_allclose(HI, damped_gram(G.reshape(S * m, n), damp), rtol=1e-12)
    np.testing.assert_allclose(HO, damped_gram(G.transpose(0, 2, 1).reshape(S * n, m), damp),
                               rtol=1e-12)


def test_sketch_b_kronecker_gradients():
    # G_s = c_s u v^T for fixed u, v: H_O ~ u u^T and H_I ~ v v^T with the stated normalisations
    rng = _rng(5)
    m, n, S = 4, 6, 9
    u, v, c = rng.standard_normal(m), rng.standard_normal(n), rng.standard_normal(S)
    G = c[:, None, None] * np.outer(u, v)[None]
    HO, HI = sketch_b(G, 0.0)
    e = np.mean(c ** 2)
    np.testing.assert_allclose(HO, e * (v @ v) / n * np.outer(u, u), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(HI, e * (u @ u) / m * np.outer(v, v), rtol=1e-12, atol=1e-14)


def test_gram_rows_is_the_gram_restricted():
    X = _rng(6).standard_normal((40, 23))
    rows = np.array([0, 5, 22, 5])
    np.testing.assert_allclose(damped_gram_rows(X, 0.03, rows), damped_gram(X, 0.03)[rows],
                               rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------- Sketch A
def test_sketch_a_zero_iterations_is_the_one_sided_start():
    rng = _rng(8)
    X, G = rng.standard_normal((50, 6)), rng.standard_normal((50, 4))
    HO, HI = sketch_a(X, G, 0, 0.01)
    np.testing.assert_allclose(HI, damped_gram(X, 0.01), rtol=1e-12)
    np.testing.assert_allclose(HO, (1 + 0.01) * np.eye(4), rtol=1e-12)


def test_sketch_a_one_iteration_by_explicit_sums():
    # the first round written out token by token: w_t = g_t g_t^T / m (H_O = I), and
    # H_O weights x_t H_1 x_t^T / |H_1|_F^2
    rng = _rng(9)
    T, n, m = 7, 3, 2
    X, G = rng.standard_normal((T, n)), rng.standard_normal((T, m))
    H1 = sum(np.outer(X[t], X[t]) for t in range(T)) / T
    HI_ref = sum(np.outer(X[t], X[t]) * (G[t] @ G[t]) / m for t in range(T)) / T
    HO_ref = sum(np.outer(G[t], G[t]) * (X[t] @ H1 @ X[t]) / np.sum(H1 * H1)
                 for t in range(T)) / T
    HO, HI = sketch_a(X, G, 1, 0.0)
    np.testing.assert_allclose(HI, HI_ref, rtol=1e-12)
    np.testing.assert_allclose(HO, HO_ref, rtol=1e-12)


def test_sketch_a_separable_tokens_keep_the_shapes():
    # every token has the same x and g: each round returns x^T x and g^T g with a scalar
    # factor, so the normalised factors are fixed points from the first round on
    rng = _rng(10)
    x, g = rng.standard_normal(5), rng.standard_normal(3)
    X, G = np.tile(x, (9, 1)), np.tile(g, (9, 1))
    for it in (1, 2, 3):
        HO, HI = sketch_a(X, G, it, 0.0)
        np.testing.assert_allclose(HI / np.linalg.norm(HI), np.outer(x, x) / np.linalg.norm(
            np.outer(x, x)), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(HO / np.linalg.norm(HO), np.outer(g, g) / np.linalg.norm(
            np.outer(g, g)), rtol=1e-12, atol=1e-14)


def test_sketch_a_scale_invariance():
    # scaling the gradients by c scales both factors of the first round by c^2: H_I through
    # its weights g H_O g^T (H_O = I), H_O through g^T g (its weights depend on X alone)
    rng = _rng(11)
    X, G = rng.standard_normal((40, 6)), rng.standard_normal((40, 4))
    HO1, HI1 = sketch_a(X, G, 1, 0.0)
    HO2, HI2 = sketch_a(X, 3.0 * G, 1, 0.0)
    np.testing.assert_allclose(HI2, 9.0 * HI1, rtol=1e-12)
    np.testing.assert_allclose(HO2, 9.0 * HO1, rtol=1e-12)
