"""fp64 CPU oracle for the BaKron solver.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import this module: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use it. It shares no code
with the CUDA path.

Sources (web pages on the method):
* [BaKron] "BaKron: Efficient Quantization with Kronecker-Factored Hessians", summary and
  abstract (insight.aitobox.com, 2026-08-07 post): two-sided adaptive rounding in the
  BoA/YAQA formulation, anti-diagonal parallelism, O(m+n) sequential steps,
  O(mn(m+n)) total work.
* [YAQA] YAQA article (news.43b.com.cn/a/479517.html):
  - section 2: the layer objective 1/2 (W-W*)^T (grad^2 L) (W-W*) with the Kronecker
    approximation grad^2 L ~ H_O (m x m) (x) H_I (n x n);
  - section 4: the rounding rule
        W_ij = Q(W*_ij + a_i^T (W*-W)[:i,:j] b_j + a_i^T (W*-W)[:i,j] + (W*-W)[i,:j] b_j),
    a_i column i of the strictly upper triangular m x m L_O, b_j column j of the strictly upper
    triangular n x n L_I, Q nearest (or stochastic) rounding;
  - section 4: the factorisation H_O = (L_O + I) D_O (L_O + I)^T (likewise H_I) and the bound
    dW (H_O (x) H_I) dW^T <= tr(D_I) tr(D_O) sigma^2;
  - section 3: the Kronecker factors themselves: the one-sided input second moment
    H_1 = E[x^T x] (also Sketch A's starting point) and Sketch B, one power-iteration round from
    the identity, (H_I)_1 = E_s[G_s^T G_s] / m and (H_O)_1 = E_s[G_s G_s^T] / n over the
    per-sequence weight gradients G_s (m x n); Sketch A, the alternating reweighted second
    moments over tokens (x_t the input row, g_t the output gradient row),
        (H_I)_i = E_t[x_t^T x_t <(H_O)_{i-1}, g_t^T g_t>] / |(H_O)_{i-1}|_F^2,
        (H_O)_i = E_t[g_t^T g_t <(H_I)_{i-1}, x_t^T x_t>] / |(H_I)_{i-1}|_F^2,
    started from (H_I)_0 = E[x^T x], (H_O)_0 = I.

Readings taken where the pages are garbled or silent (each one is listed in the design notes):
* index ranges ``:i`` / ``:j`` are exclusive (rows k < i, columns l < j);
* L is strictly *upper* triangular, so H = (I+L) D (I+L)^T is a U D U^T factorisation
  (the section-4 text also calls it "unit lower"; only the upper reading makes the rule causal
  and the bound hold);
* Q is round-half-to-even of pre/s_i followed by a clamp to [-2^(b-1), 2^(b-1)-1], per-row
  scale s_i; s_i = 0 gives code 0. The pages fix no precision for this integer decision, so it
  is the plain one: the real quotient pre/s_i, formed here as one fp64 division of the fp64
  pre by the (fp32) scale. For inputs that are fp32 values (identity factors, where pre = W*)
  this decides exactly: a nonzero distance between pre/s and a half-integer is then far above
  the fp64 rounding of the quotient;
* E = W* - W always includes the clamp error;
* the proxy loss is tr(H_O dW H_I dW^T) with no factor 1/2;
* the base quantizer is pluggable ([BaKron] summary: the solver is modular in the base
  quantizer): the grid step may be per row and column group, s_ij = scales[i, j // group_size],
  and Q may round to a sorted scalar codebook c_0 < ... < c_{K-1} instead of the integers:
  the quantizer is given by its decision thresholds, the fp32 midpoints
  mu_k = fl32((c_k + c_{k+1}) / 2): the code is the number of thresholds strictly below the
  quotient x = pre / s_ij (real, as for the integer grid), a tie going to the lower entry, and
  W_ij = s_ij c_code;
* incoherence processing ([YAQA] section 4: like LDLQ, lower the incoherence of the Hessian
  factors before quantising) is the randomised Hadamard transform T_d = H_d S_d / sqrt(d) on
  both sides: W~ = T_m W* T_n^T, H_O~ = T_m H_O T_m^T, H_I~ = T_n H_I T_n^T, and after
  rounding W = T_m^T W~_q T_n. H_d is Sylvester's for d = 2^k and the Kronecker product
  H_28 (x) H_{2^k} for d = 28 2^k, with H_28 Paley's skew construction over GF(27) =
  GF(3)[t] / (t^3 + 2t + 1), element e <-> (e mod 3) + (e div 3 mod 3) t + (e div 9) t^2,
  H_28[0][*] = 1, H_28[1+x][0] = -1, H_28[1+x][1+y] = chi(x - y) + [x = y] (chi the
  quadratic character); the signs S_d are bit i mod 256 of the Philox4x64-10 block keyed
  (seed, 0) at counter (i div 256, 0, 1, 0) (word (i mod 256) div 64, bit i mod 64; set
  bit = -1);
* every Kronecker factor is damped like the benchmark's inputs: H + damp * mean(diag(H)) * I,
  the mean taken over the undamped diagonal;
* stochastic Q (the section-4 alternative to nearest rounding) rounds x = pre/s_i up with
  probability frac(x): code = clamp(floor(x + u)) with u uniform on (0, 1). The pages name no
  generator, so u is drawn by Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
  numbers: as easy as 1, 2, 3", SC 2011), keyed by (seed, 0) with counter (j // 16, i, 0, 0);
  entry (i, j) takes the 16-bit field j % 16 of the 256-bit block (word (j % 16) // 4, bits
  16 (j % 4) and up), u = (field + 1/2) / 2^16. x is the real quotient as for nearest
  rounding, and x + u is formed in fp64 (u has 17 significant bits, so the sum is the real
  one to fp64 precision).

Parity status: every function below is pinned against things other than itself by
``tests/test_oracle.py`` (factorisation, rule, loss), ``test_oracle_stochastic.py`` (Philox and
stochastic Q), ``test_oracle_hessian.py`` (the Kronecker factors), ``test_oracle_quantizer.py``
(per-group steps, codebooks) and ``test_oracle_incoherence.py`` (the Hadamard transform):
closed forms, library routines (numpy Cholesky and Philox, scipy's Hadamard matrix), a
different algorithm (GPTQ in its optimal-brain-surgeon form on the vectorised problem),
special cases and brute force. No worked numerical example is printed on the pages, so there
is no golden value from the pages themselves.
"""
from __future__ import annotations

import itertools

import numpy as np

__all__ = [
    "udu", "quantize", "round_naive", "round_row_sweep", "fixed_point_pre",
    "proxy_loss", "proxy_loss_kron", "brute_force_fixed_points", "gptq_obs",
    "code_range", "fixed_point_pre_rows", "band_check", "grid_quotient",
    "philox4x64_10", "dither", "quantize_stochastic", "damped_gram", "sketch_b",
    "damped_gram_rows", "codebook_midpoints", "quantize_codebook", "scale_of", "sketch_a",
    "gf27_chi", "hadamard28", "hadamard", "rht_signs", "rht_matrix", "rht", "hadamard_rows",
]


def code_range(bits: int) -> tuple[int, int]:
    return -(1 << (bits - 1)), (1 << (bits - 1)) - 1


# ---------------------------------------------------------------------------------------------
# Factorisation: H = (I + L) D (I + L)^T, L strictly upper triangular ([YAQA] section 4).
# ---------------------------------------------------------------------------------------------
def udu(H: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Textbook U D U^T factorisation, last index first, in fp64.

    For j = d-1 down to 0:
        D_j      = H_jj - sum_{k>j} U_jk^2 D_k
        U_ij     = (H_ij - sum_{k>j} U_ik U_jk D_k) / D_j      for i < j
    with U = I + L. Returns (L, D): L strictly upper (zeros on and below the diagonal).
    Raises ValueError on a non-positive or non-finite pivot.
    """
    H = np.asarray(H, dtype=np.float64)
    d = H.shape[0]
    U = np.eye(d)
    D = np.zeros(d)
    for j in range(d - 1, -1, -1):
        tail = slice(j + 1, d)
        D[j] = H[j, j] - np.dot(U[j, tail] ** 2, D[tail])
        if not np.isfinite(D[j]) or D[j] <= 0.0:
            raise ValueError(f"non-positive pivot at index {j}: {D[j]}")
        if j > 0:
            U[:j, j] = (H[:j, j] - U[:j, tail] @ (U[j, tail] * D[tail])) / D[j]
    L = U - np.eye(d)
    return L, D


# ---------------------------------------------------------------------------------------------
# Base quantizer Q ([YAQA] section 4: nearest rounding; reading: half-even, then clamp).
# ---------------------------------------------------------------------------------------------
def grid_quotient(pre, s):
    """The quotient pre / s on which Q decides: the real quotient, formed as one fp64 division
    (elementwise on arrays)."""
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.asarray(pre, dtype=np.float64) / np.asarray(s, dtype=np.float64)
    return q


def quantize(pre: float, s: float, bits: int) -> int:
    """Code for one entry: clamp(round_half_even(pre / s)); s == 0 gives 0."""
    lo, hi = code_range(bits)
    if s == 0.0:
        return 0
    c = float(np.rint(grid_quotient(pre, s)))
    return int(min(max(c, lo), hi))


# ---------------------------------------------------------------------------------------------
# Stochastic Q ([YAQA] section 4 allows stochastic rounding in place of nearest rounding).
# ---------------------------------------------------------------------------------------------
_M64 = (1 << 64) - 1
_PHILOX_M = (0xD2E7470EE14C6C93, 0xCA5A826395121157)   # round multipliers of Philox4x64
_PHILOX_W = (0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B)   # key increments (Weyl sequence)


def philox4x64_10(counter, key):
    """Philox4x64 with 10 rounds (Salmon et al., SC 2011, section 4): per round the two
    64 x 64 -> 128-bit products of words 0 and 2 with the round multipliers, the high halves
    xored with words 1 and 3 and the round key, the words permuted; the key advances by the
    Weyl increments between rounds. counter: 4 ints < 2^64, key: 2 ints < 2^64. Returns the
    4 output words."""
    x0, x1, x2, x3 = (int(v) & _M64 for v in counter)
    k0, k1 = (int(v) & _M64 for v in key)
    for _ in range(10):
        p0 = _PHILOX_M[0] * x0
        p1 = _PHILOX_M[1] * x2
        x0, x1, x2, x3 = (p1 >> 64) ^ x1 ^ k0, p1 & _M64, (p0 >> 64) ^ x3 ^ k1, p0 & _M64
        k0 = (k0 + _PHILOX_W[0]) & _M64
        k1 = (k1 + _PHILOX_W[1]) & _M64
    return x0, x1, x2, x3


def dither(rows, n: int, seed: int) -> np.ndarray:
    """The uniform variates u_ij of stochastic Q for the given rows (an int m gives rows
    0..m-1), all n columns: len(rows) x n fp64, each (k + 1/2) / 2^16 for a 16-bit k."""
    rows = np.arange(rows) if np.isscalar(rows) else np.asarray(rows)
    out = np.empty((rows.size, n))
    for a, i in enumerate(rows):
        for cb in range((n + 15) // 16):
            words = philox4x64_10((cb, int(i), 0, 0), (seed, 0))
            for t in range(min(16, n - 16 * cb)):
                k = (words[t // 4] >> (16 * (t % 4))) & 0xFFFF
                out[a, 16 * cb + t] = (k + 0.5) / 65536.0
    return out


def quantize_stochastic(pre: float, s: float, bits: int, u: float) -> int:
    """Stochastic code for one entry: clamp(floor(x + u)), x the quotient pre / s and x + u
    both in fp64; s == 0 gives 0."""
    lo, hi = code_range(bits)
    if s == 0.0:
        return 0
    y = float(grid_quotient(pre, s)) + float(u)
    return int(min(max(float(np.floor(y)), lo), hi))


# ---------------------------------------------------------------------------------------------
# Pluggable base quantizer ([BaKron] summary): per-group grid steps, scalar codebooks.
# ---------------------------------------------------------------------------------------------
def codebook_midpoints(codebook) -> np.ndarray:
    """The decision thresholds of a sorted codebook: fl32((c_k + c_{k+1}) / 2) (fp32 sum and
    halving, both exact or correctly rounded), returned as fp64."""
    c = np.asarray(codebook, dtype=np.float32)
    return ((c[:-1] + c[1:]) * np.float32(0.5)).astype(np.float64)


def quantize_codebook(pre: float, s: float, codebook) -> int:
    """Index of the nearest codebook entry to the quotient pre / s: the number of fp32
    midpoints strictly below it (a tie goes to the lower entry); s == 0 gives index 0."""
    if s == 0.0:
        return 0
    x = float(grid_quotient(pre, s))
    return int(np.sum(x > codebook_midpoints(codebook)))


def scale_of(scales, i: int, j: int, group_size=None) -> float:
    """The grid step of entry (i, j): scales[i] (one per row) or scales[i, j // group_size]."""
    sc = np.asarray(scales)
    return float(sc[i]) if sc.ndim == 1 else float(sc[i, j // group_size])


def _q(pre, s, bits, U, i, j, codebook=None):
    if codebook is not None:
        return quantize_codebook(pre, s, codebook)
    return quantize(pre, s, bits) if U is None else quantize_stochastic(pre, s, bits, U[i, j])


def _value(code, s, codebook=None):
    return s * (code if codebook is None else float(np.float32(codebook[code])))


# ---------------------------------------------------------------------------------------------
# The rule, entry by entry, in raster order ([YAQA] section 4). Raster order is a valid order
# because entry (i, j) reads only entries (k, l) with k <= i and l <= j, (k, l) != (i, j).
# ---------------------------------------------------------------------------------------------
def round_naive(Wstar, L_O, L_I, scales, bits, return_pre=False, dither=None, codebook=None,
                group_size=None):
    """Plain definition, O(m^2 n^2 / 4) multiply-adds.

    pre_ij = W*_ij + a_i^T E[:i,:j] b_j + a_i^T E[:i,j] + E[i,:j] b_j,   E = W* - W
    with a_i = L_O[:i, i] and b_j = L_I[:j, j]. ``dither`` (m x n variates u_ij) selects
    stochastic Q; None selects nearest rounding. ``codebook`` selects the nearest entry of a
    sorted codebook (codes are then entry indices); 2-D ``scales`` (m x G) are per row and
    column group of ``group_size`` columns.
    Returns (codes int64 m x n, W fp64 m x n[, pre fp64 m x n]).
    """
    Ws = np.asarray(Wstar, dtype=np.float64)
    LO = np.asarray(L_O, dtype=np.float64)
    LI = np.asarray(L_I, dtype=np.float64)
    s = np.asarray(scales, dtype=np.float64)
    m, n = Ws.shape
    E = np.zeros((m, n))
    W = np.zeros((m, n))
    C = np.zeros((m, n), dtype=np.int64)
    P = np.zeros((m, n))
    for i in range(m):
        a = LO[:i, i]
        for j in range(n):
            b = LI[:j, j]
            pre = Ws[i, j]
            if i > 0 and j > 0:
                pre += (a @ E[:i, :j]) @ b
            if i > 0:
                pre += a @ E[:i, j]
            if j > 0:
                pre += E[i, :j] @ b
            sij = scale_of(s, i, j, group_size)
            c = _q(pre, sij, bits, dither, i, j, codebook)
            C[i, j] = c
            W[i, j] = _value(c, sij, codebook)
            E[i, j] = Ws[i, j] - W[i, j]
            P[i, j] = pre
    return (C, W, P) if return_pre else (C, W)


def round_row_sweep(Wstar, L_O, L_I, scales, bits, return_pre=False, dither=None, codebook=None,
                    group_size=None):
    """Same result as ``round_naive`` in O(mn(m+n)) work (the row-by-row reading).

    Row i sees every earlier row only through T_i = sum_{k<i} L_O[k,i] E_k (a row vector).
    Substituting into the rule gives pre_ij = r_j + sum_{l<j} E_il L_I[l,j] with
    r = W*_i + T_i + T_i L_I, i.e. one-sided LDLQ of the biased row (a left-to-right pass).
    """
    Ws = np.asarray(Wstar, dtype=np.float64)
    LO = np.asarray(L_O, dtype=np.float64)
    LI = np.asarray(L_I, dtype=np.float64)
    s = np.asarray(scales, dtype=np.float64)
    m, n = Ws.shape
    E = np.zeros((m, n))
    W = np.zeros((m, n))
    C = np.zeros((m, n), dtype=np.int64)
    P = np.zeros((m, n))
    for i in range(m):
        T = LO[:i, i] @ E[:i, :] if i > 0 else np.zeros(n)
        r = Ws[i] + T + T @ LI
        for j in range(n):
            pre = r[j] + E[i, :j] @ LI[:j, j]
            sij = scale_of(s, i, j, group_size)
            c = _q(pre, sij, bits, dither, i, j, codebook)
            C[i, j] = c
            W[i, j] = _value(c, sij, codebook)
            E[i, j] = Ws[i, j] - W[i, j]
            P[i, j] = pre
    return (C, W, P) if return_pre else (C, W)


def fixed_point_pre(Wstar, W, L_O, L_I):
    """Closed form of the pre-rounding values given the final W:

        pre = W* + (I + L_O)^T E (I + L_I) - E,    E = W* - W,

    evaluated with fp64 matrix products. Because (I + L_O)^T is lower and (I + L_I) upper
    triangular, entry (i, j) only sees E_kl with k <= i, l <= j; the -E removes the (i, j)
    self-term. A correct solve satisfies W_ij = Q(pre_ij) at every entry.
    """
    Ws = np.asarray(Wstar, dtype=np.float64)
    E = Ws - np.asarray(W, dtype=np.float64)
    m, n = E.shape
    Ao = np.eye(m) + np.asarray(L_O, dtype=np.float64)
    Ai = np.eye(n) + np.asarray(L_I, dtype=np.float64)
    return Ws + (Ao.T @ E) @ Ai - E


def fixed_point_pre_rows(Wstar, W, L_O, L_I, rows):
    """``fixed_point_pre`` restricted to the given rows (same closed form, fp64):
    pre[R] = W*[R] + ((I + L_O)^T)[R, :] E (I + L_I) - E[R]."""
    rows = np.asarray(rows)
    Ws = np.asarray(Wstar, dtype=np.float64)
    E = Ws - np.asarray(W, dtype=np.float64)
    m, n = E.shape
    LI = np.asarray(L_I, dtype=np.float64)
    AoT_R = np.asarray(np.asarray(L_O)[:, rows], dtype=np.float64).T.copy()   # (L_O^T)[R, :]
    AoT_R[np.arange(rows.size), rows] += 1.0
    T = AoT_R @ E
    return Ws[rows] + T + T @ LI - E[rows]


def band_check(pre, codes, scales, bits, band=1e-3, dither=None, codebook=None, group_size=None):
    """Compare codes with Q(pre) under the exemption band of the tolerance rule.

    An entry may disagree only if pre/s lies within ``band`` grid steps of a rounding boundary
    (a half-integer for nearest rounding; for stochastic Q with variates ``dither``, an
    integer value of pre/s + u; for a codebook, a midpoint of two entries). 2-D ``scales``
    are per row and column group. Returns (n_mismatch, n_mismatch_outside_band, n_in_band).
    """
    s = np.asarray(scales, dtype=np.float64)
    if s.ndim == 1:
        s = s[:, None]
    else:
        s = np.repeat(s, group_size, axis=1)[:, :pre.shape[1]]
    lo, hi = code_range(bits)
    s_safe = np.where(s > 0, s, 1.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        x = np.where(s > 0, pre / s_safe, 0.0)
    xq = np.where(s > 0, grid_quotient(pre, np.broadcast_to(s_safe, pre.shape)), 0.0)
    if codebook is not None:
        mids = codebook_midpoints(codebook)
        q = np.sum(xq[..., None] > mids, axis=-1).astype(np.float64)
        frac = np.min(np.abs(x[..., None] - mids), axis=-1)
    elif dither is None:
        q = np.clip(np.rint(xq), lo, hi)
        frac = np.abs(x - np.floor(x) - 0.5)
    else:
        u = np.asarray(dither, dtype=np.float64)
        q = np.clip(np.floor(xq + u), lo, hi)
        frac = np.abs(x + u - np.rint(x + u))
    q = np.where(s > 0, q, 0.0)
    in_band = frac < band
    mism = q != np.asarray(codes, dtype=np.float64)
    return int(mism.sum()), int((mism & ~in_band).sum()), int(in_band.sum())


def proxy_loss(dW, H_O, H_I) -> float:
    """tr(H_O dW H_I dW^T) in fp64 ([YAQA] section 4 proxy; no factor 1/2), the trace of the
    product written out: tr(A dW^T) = sum_ij A_ij dW_ij with A = H_O dW H_I."""
    d = np.asarray(dW, dtype=np.float64)
    A = np.asarray(H_O, np.float64) @ d @ np.asarray(H_I, np.float64)
    return float(np.sum(A * d))


def proxy_loss_kron(dW, H_O, H_I) -> float:
    """vec(dW)^T (H_O (x) H_I) vec(dW) with row-major vec, by the explicit Kronecker product
    (tiny shapes only)."""
    v = np.asarray(dW, dtype=np.float64).reshape(-1)
    K = np.kron(np.asarray(H_O, np.float64), np.asarray(H_I, np.float64))
    return float(v @ K @ v)


# ---------------------------------------------------------------------------------------------
# Incoherence processing ([YAQA] section 4): the randomised Hadamard transform.
# ---------------------------------------------------------------------------------------------
def _gf27(e: int) -> tuple[int, int, int]:
    return e % 3, (e // 3) % 3, e // 9


def _gf27_mul(a, b):
    """Product in GF(3)[t] / (t^3 + 2t + 1), i.e. t^3 = t + 2 (coefficients mod 3)."""
    c = [0] * 5
    for i in range(3):
        for j in range(3):
            c[i + j] += a[i] * b[j]
    for k in (4, 3):                       # t^k = t^(k-3) (t + 2)
        c[k - 2] += c[k]
        c[k - 3] += 2 * c[k]
        c[k] = 0
    return tuple(v % 3 for v in c[:3])


def gf27_chi() -> np.ndarray:
    """The quadratic character of GF(27) on the 27 labelled elements: 0, +1 (nonzero square)
    or -1."""
    squares = {_gf27_mul(_gf27(e), _gf27(e)) for e in range(1, 27)}
    return np.array([0] + [1 if _gf27(e) in squares else -1 for e in range(1, 27)])


def hadamard28() -> np.ndarray:
    """Paley's skew Hadamard matrix of order 28 (q = 27), rows/columns 1 + x for x in GF(27)."""
    chi = gf27_chi()
    H = np.zeros((28, 28))
    H[0, :] = 1.0
    H[1:, 0] = -1.0
    for x in range(27):
        for y in range(27):
            a, b = _gf27(x), _gf27(y)
            diff = sum(((a[k] - b[k]) % 3) * 3 ** k for k in range(3))
            H[1 + x, 1 + y] = chi[diff] + (1.0 if x == y else 0.0)
    return H


def hadamard(d: int) -> np.ndarray:
    """H_d for d = 2^k (Sylvester: (-1)^popcount(i & j)) or d = 28 2^k (H_28 (x) H_{2^k})."""
    k = d // 28 if d % 28 == 0 and (d // 28) & (d // 28 - 1) == 0 else d
    if k & (k - 1) != 0:
        raise ValueError(f"no Hadamard construction here for d = {d}")
    i = np.arange(k)
    syl = np.array([[(-1.0) ** bin(a & b).count("1") for b in i] for a in i])
    return syl if k == d else np.kron(hadamard28(), syl)


def hadamard_rows(d: int, rows) -> np.ndarray:
    """Rows ``rows`` of H_d without forming H_d (the same definitions: Sylvester's
    (-1)^popcount(i & j), times H_28[i div 2^k][j div 2^k] for d = 28 2^k)."""
    rows = np.asarray(rows)
    k = d // 28 if d % 28 == 0 and (d // 28) & (d // 28 - 1) == 0 else d
    if k & (k - 1) != 0:
        raise ValueError(f"no Hadamard construction here for d = {d}")
    j = np.arange(d)
    b_i, b_j = (rows % k)[:, None], (j % k)[None, :]
    par = np.vectorize(lambda v: bin(int(v)).count("1") & 1)(b_i & b_j)
    out = np.where(par == 1, -1.0, 1.0)
    if k != d:
        out = out * hadamard28()[(rows // k)[:, None], (j // k)[None, :]]
    return out


def rht_signs(d: int, seed: int) -> np.ndarray:
    """The random signs S_d (+1 / -1) of the transform."""
    out = np.empty(d)
    for blk in range((d + 255) // 256):
        words = philox4x64_10((blk, 0, 1, 0), (seed, 0))
        for t in range(min(256, d - 256 * blk)):
            out[256 * blk + t] = -1.0 if (words[t // 64] >> (t % 64)) & 1 else 1.0
    return out


def rht_matrix(d: int, seed: int) -> np.ndarray:
    """T_d = H_d diag(S_d) / sqrt(d), orthogonal, in fp64."""
    return hadamard(d) * rht_signs(d, seed)[None, :] / np.sqrt(d)


def rht(X, seed_rows: int, seed_cols: int, inverse: bool = False) -> np.ndarray:
    """T_r X T_c^T (or, inverse, T_r^T X T_c) for X (r x c), in fp64."""
    X = np.asarray(X, dtype=np.float64)
    Tr, Tc = rht_matrix(X.shape[0], seed_rows), rht_matrix(X.shape[1], seed_cols)
    return Tr.T @ X @ Tc if inverse else Tr @ X @ Tc.T


# ---------------------------------------------------------------------------------------------
# The Kronecker factors ([YAQA] section 3), damped.
# ---------------------------------------------------------------------------------------------
def _damp(G: np.ndarray, damp: float) -> np.ndarray:
    H = G.copy()
    H[np.diag_indices_from(H)] += damp * float(np.mean(np.diag(G)))
    return H


def damped_gram(X, damp: float) -> np.ndarray:
    """E[x^T x] over the N rows x of X (N x d), plus damp * mean(diag) * I, in fp64:
    H = X^T X / N + damp * mean_i (X^T X / N)_ii * I."""
    X = np.asarray(X, dtype=np.float64)
    return _damp(X.T @ X / X.shape[0], damp)


def damped_gram_rows(X, damp: float, rows) -> np.ndarray:
    """``damped_gram`` restricted to the given rows (same definition, fp64): the rows R of
    X^T X / N, with damp * mean of the full diagonal added at (R[k], R[k])."""
    X = np.asarray(X, dtype=np.float64)
    rows = np.asarray(rows)
    N = X.shape[0]
    out = X[:, rows].T @ X / N
    mean_diag = float(np.mean(np.einsum("ti,ti->i", X, X))) / N
    out[np.arange(rows.size), rows] += damp * mean_diag
    return out


def sketch_a(X, G, iterations: int, damp: float) -> tuple[np.ndarray, np.ndarray]:
    """Sketch A: ``iterations`` rounds of the alternating update from (H_I)_0 = E[x^T x],
    (H_O)_0 = I over the token rows of X (T x n, inputs) and G (T x m, output gradients), both
    factors of a round computed from the previous round's pair; the returned pair is damped
    (the iterations use the undamped factors). Returns (H_O, H_I) in fp64."""
    X = np.asarray(X, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    T = X.shape[0]
    HI = X.T @ X / T
    HO = np.eye(G.shape[1])
    for _ in range(iterations):
        w_in = np.einsum("ta,ab,tb->t", G, HO, G) / np.sum(HO * HO)    # <H_O, g^T g> / |H_O|^2
        w_out = np.einsum("ta,ab,tb->t", X, HI, X) / np.sum(HI * HI)   # <H_I, x^T x> / |H_I|^2
        HI, HO = (X * w_in[:, None]).T @ X / T, (G * w_out[:, None]).T @ G / T
    return _damp(HO, damp), _damp(HI, damp)


def sketch_b(G, damp: float) -> tuple[np.ndarray, np.ndarray]:
    """Sketch B, one power-iteration round from H_O = H_I = I, for per-sequence gradients
    G (S x m x n), each factor damped: returns (H_O, H_I) with
    H_O = (1/S) sum_s G_s G_s^T / n,   H_I = (1/S) sum_s G_s^T G_s / m."""
    G = np.asarray(G, dtype=np.float64)
    S, m, n = G.shape
    HO = sum(G[s] @ G[s].T for s in range(S)) / (S * n)
    HI = sum(G[s].T @ G[s] for s in range(S)) / (S * m)
    return _damp(HO, damp), _damp(HI, damp)


# ---------------------------------------------------------------------------------------------
# Independent algorithms used only to pin the rule.
# ---------------------------------------------------------------------------------------------
def gptq_obs(w_star: np.ndarray, H: np.ndarray, scales: np.ndarray, bits: int, dither=None,
             codebook=None):
    """GPTQ in its optimal-brain-surgeon form on a vector w (length N) with Hessian H.

    Coordinates are fixed in index order. After fixing coordinate q to its quantised value,
    every still-free coordinate f moves by  -(w_q - Q(w_q)) [H_F^{-1}]_{f q} / [H_F^{-1}]_{q q},
    where H_F is H restricted to the free set (q included). ``scales[q]`` is the grid step of
    coordinate q; ``dither`` (length N) selects stochastic Q. Returns integer codes. Uses an
    explicit inverse per step: tiny N only.
    """
    w = np.asarray(w_star, dtype=np.float64).copy()
    H = np.asarray(H, dtype=np.float64)
    N = w.shape[0]
    codes = np.zeros(N, dtype=np.int64)
    for q in range(N):
        if codebook is not None:
            c = quantize_codebook(w[q], float(scales[q]), codebook)
        elif dither is None:
            c = quantize(w[q], float(scales[q]), bits)
        else:
            c = quantize_stochastic(w[q], float(scales[q]), bits, float(dither[q]))
        codes[q] = c
        wq = _value(c, float(scales[q]), codebook)
        F = np.arange(q, N)
        Hinv = np.linalg.inv(H[np.ix_(F, F)])
        delta = (w[q] - wq) / Hinv[0, 0]
        w[F] -= delta * Hinv[:, 0]
        w[q] = wq
    return codes


def brute_force_fixed_points(Wstar, L_O, L_I, scales, bits, chunk=4096, dither=None,
                             codebook=None):
    """All code matrices C with C = Q(pre(C)) under the closed form, by enumeration.

    Every candidate C in [lo, hi]^(m x n) is tried: W = s * C, pre is the closed form of
    ``fixed_point_pre`` (evaluated for a batch of candidates at once with the same fp64
    products), and C is kept when Q(pre) == C at every entry (nearest, stochastic with the
    variates ``dither``, or the index of the nearest ``codebook`` entry, when the candidates
    are the indices 0 .. K-1 and W = s * c_C). Tiny shapes only
    ((2^bits)^(mn) candidates). Rows with s_i = 0 are not supported here.
    """
    Ws = np.asarray(Wstar, dtype=np.float64)
    s = np.asarray(scales, dtype=np.float64)
    m, n = Ws.shape
    lo, hi = code_range(bits)
    Ao = np.eye(m) + np.asarray(L_O, dtype=np.float64)
    Ai = np.eye(n) + np.asarray(L_I, dtype=np.float64)
    values = np.arange(lo, hi + 1) if codebook is None else np.arange(len(codebook))
    cb32 = None if codebook is None else np.asarray(codebook, dtype=np.float32).astype(np.float64)
    total = len(values) ** (m * n)
    found = []
    for start in range(0, total, chunk):
        idx = np.arange(start, min(start + chunk, total))
        digits = np.empty((idx.size, m * n), dtype=np.int64)
        rest = idx.copy()
        for p in range(m * n - 1, -1, -1):
            digits[:, p] = values[rest % len(values)]
            rest //= len(values)
        C = digits.reshape(-1, m, n)
        E = Ws[None] - s[None, :, None] * (C if cb32 is None else cb32[C])
        pre = Ws[None] + np.einsum("ki,bkl,lj->bij", Ao, E, Ai) - E
        xq = grid_quotient(pre, np.broadcast_to(s[None, :, None], pre.shape))
        if codebook is not None:
            Q = np.sum(xq[..., None] > codebook_midpoints(codebook), axis=-1)
        elif dither is None:
            Q = np.clip(np.rint(xq), lo, hi)
        else:
            u = np.asarray(dither, dtype=np.float64)[None]
            Q = np.clip(np.floor(xq + u), lo, hi)
        ok = np.all(Q == C, axis=(1, 2))
        found.extend(C[ok])
    return found
