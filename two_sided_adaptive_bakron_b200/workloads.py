"""Seeded synthetic inputs for the BaKron solver (layer-shaped W*, damped Kronecker factors).

This module only *draws* inputs. It holds none of the solver's arithmetic (no factorisation,
no rounding, no loss), so that both the CPU oracle (under ``oracle/``) and the CUDA path can
consume the very same arrays.

Recipe (one seeded ``numpy.random.Generator(PCG64(seed))`` per workload; seed = workload id
unless given). Draw order: W*, outlier column indices, the token matrix X (+ its per-column
scales), then the gradient factors Z, B and the isotropic noise.

* W* (m x n, out x in): N(0, 1/n) drawn in fp64 and cast to fp32, or Student-t(5)/sqrt(n);
  optional outlier input columns multiplied by a constant factor.
* H_I (n x n) = X^T X / N + 0.01 * mean(diag(X^T X / N)) * I, X an N x n Gaussian token matrix
  (fp32 draws), with per-column log-normal(0, 1) scales or the same outlier columns scaled.
* H_O (m x m) = G^T G / N + the same relative damping, where G is either built like X
  (per-column log-normal scales) or is a rank-r gradient sketch
  G = Z (N x r) B (r x m) / sqrt(r) + 0.1 * noise (N x m).
* Per-row scales s_i = max_j |W*_ij| / (2^(bits-1) - 0.5), in fp32; codes lie in
  [-2^(bits-1), 2^(bits-1) - 1].

The Kronecker factor orientation H ~ H_O (output, m x m) (x) H_I (input, n x n) follows the YAQA
article (news.43b.com.cn), section 2 "YAQA: a global view", Kronecker approximation of the
Fisher; the Gram construction with relative damping follows the workload definitions of the
BaKron solver benchmark (synthetic LLM layer shapes).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = ["Workload", "WORKLOADS", "make_workload", "make_layer_samples", "row_scales",
           "damped_gram", "code_range"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and statistics of one synthetic layer."""
    name: str
    m: int                      # output features (rows of W*)
    n: int                      # input features (cols of W*)
    bits: int                   # code width
    wdist: str = "gauss"        # "gauss" | "student5"
    n_outliers: int = 0         # number of outlier input columns (W* and X share them)
    outlier_scale: float = 1.0
    tokens: int = 512           # rows of X
    x_lognormal: bool = True    # per-column log-normal(0,1) scales on X
    grad_rows: int = 512        # rows of G
    grad_rank: int = 0          # 0: G built like X (Gaussian x log-normal columns)
    damp: float = 0.01
    seed: int = 0
    variant: str = "kron"       # "kron" | "ho_identity" | "identity"


# The five layer workloads. Shapes stand in for LLM projections: 8B-class attention
# (4096 x 4096), 8B-class down-projection (4096 x 14336), 70B-class up/gate (28672 x 8192).
WORKLOADS = {
    "small_64x128": Workload("small_64x128", 64, 128, 4, tokens=512, grad_rows=512, seed=0),
    "small_64x128_ho_identity": Workload("small_64x128_ho_identity", 64, 128, 4, tokens=512,
                                         grad_rows=512, seed=0, variant="ho_identity"),
    "small_64x128_identity": Workload("small_64x128_identity", 64, 128, 4, tokens=512,
                                      grad_rows=512, seed=0, variant="identity"),
    "sq_1024": Workload("sq_1024", 1024, 1024, 2, tokens=2048, grad_rows=2048, grad_rank=32,
                        seed=1),
    "attn_4096": Workload("attn_4096", 4096, 4096, 2, n_outliers=8, outlier_scale=20.0,
                          tokens=4096, x_lognormal=False, grad_rows=4096, grad_rank=64, seed=2),
    "down_4096x14336": Workload("down_4096x14336", 4096, 14336, 3, wdist="student5",
                                tokens=8192, grad_rows=8192, grad_rank=128, seed=3),
    "upgate_28672x8192": Workload("upgate_28672x8192", 28672, 8192, 2, n_outliers=16,
                                  outlier_scale=10.0, tokens=8192, x_lognormal=False,
                                  grad_rows=16384, grad_rank=256, seed=4),
}


def code_range(bits: int) -> tuple[int, int]:
    """Signed code range [-2^(bits-1), 2^(bits-1)-1]."""
    return -(1 << (bits - 1)), (1 << (bits - 1)) - 1


def row_scales(Wstar: np.ndarray, bits: int) -> np.ndarray:
    """Per-row max-abs scales s_i = max|W*_i| / (2^(bits-1) - 0.5), computed in fp32."""
    w = np.asarray(Wstar, dtype=np.float32)
    denom = np.float32((1 << (bits - 1)) - 0.5)
    return (np.abs(w).max(axis=1) / denom).astype(np.float32)


def _gram(Xf32: np.ndarray, device: Optional[str]) -> np.ndarray:
    """X^T X / N in fp64 (torch on ``device`` when given, numpy otherwise)."""
    N = Xf32.shape[0]
    if device is not None:
        import torch
        xt = torch.from_numpy(Xf32).to(device=device, dtype=torch.float64)
        g = (xt.T @ xt) / N
        out = g.cpu().numpy()
        del xt, g
        return out
    x = Xf32.astype(np.float64)
    return (x.T @ x) / N


def damped_gram(Xf32: np.ndarray, damp: float, device: Optional[str] = None) -> np.ndarray:
    """Damped Gram matrix X^T X / N + damp * mean(diag) * I, returned as fp32."""
    g = _gram(Xf32, device)
    g = 0.5 * (g + g.T)
    g[np.diag_indices_from(g)] += damp * float(np.mean(np.diag(g)))
    return g.astype(np.float32)


def _token_matrix(rng, N: int, d: int, lognormal: bool, out_idx, out_scale):
    X = rng.standard_normal((N, d), dtype=np.float32)
    if lognormal:
        X *= np.exp(rng.standard_normal(d)).astype(np.float32)[None, :]
    if out_idx is not None and len(out_idx):
        X[:, out_idx] *= np.float32(out_scale)
    return X


def make_layer_samples(w: Workload | str, seed: Optional[int] = None):
    """Draw (W*, X, G, scales, bits): the layer and the raw samples whose damped second moments
    are its Kronecker factors, all fp32 numpy arrays. X (tokens x n) gives H_I, G (gradient
    rows x m) gives H_O; either is None where the workload's factor is the identity. The draws
    are those of ``make_workload`` (same order), which forms the damped Grams from them.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    m, n = w.m, w.n
    if w.wdist == "gauss":
        Wstar = rng.standard_normal((m, n)) / math.sqrt(n)
    elif w.wdist == "student5":
        Wstar = rng.standard_t(5.0, size=(m, n)) / math.sqrt(n)
    else:
        raise ValueError(w.wdist)
    out_idx = None
    if w.n_outliers:
        out_idx = np.sort(rng.choice(n, size=w.n_outliers, replace=False))
        Wstar[:, out_idx] *= w.outlier_scale
    Wstar = Wstar.astype(np.float32)

    X = None
    if w.variant != "identity":
        X = _token_matrix(rng, w.tokens, n, w.x_lognormal, out_idx, w.outlier_scale)

    G = None
    if w.variant in ("identity", "ho_identity"):
        pass
    elif w.grad_rank == 0:
        G = _token_matrix(rng, w.grad_rows, m, True, None, 1.0)
    else:
        r = w.grad_rank
        Z = rng.standard_normal((w.grad_rows, r), dtype=np.float32)
        B = rng.standard_normal((r, m), dtype=np.float32)
        G = (Z @ B) * np.float32(1.0 / math.sqrt(r))
        G += np.float32(0.1) * rng.standard_normal((w.grad_rows, m), dtype=np.float32)
        del Z, B

    return Wstar, X, G, row_scales(Wstar, w.bits), w.bits


def make_workload(w: Workload | str, device: Optional[str] = None, seed: Optional[int] = None):
    """Draw (W*, H_O, H_I, scales, bits) for a workload, all fp32 numpy arrays.

    ``device`` (e.g. "cuda") only moves the fp64 Gram products onto a GPU for speed; the random
    draws are always numpy PCG64 on the host.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    Wstar, X, G, scales, bits = make_layer_samples(w, seed)
    H_I = np.eye(w.n, dtype=np.float32) if X is None else damped_gram(X, w.damp, device)
    del X
    H_O = np.eye(w.m, dtype=np.float32) if G is None else damped_gram(G, w.damp, device)
    del G
    return Wstar, H_O, H_I, scales, bits


def random_problem(m: int, n: int, bits: int, seed: int, tokens: Optional[int] = None,
                   kind: str = "kron"):
    """Small random problem of arbitrary shape (tests: ragged and degenerate shapes).

    kind: "kron" (both factors damped Grams), "ho_identity", "hi_identity", "identity".
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    Wstar = (rng.standard_normal((m, n)) / math.sqrt(max(n, 1))).astype(np.float32)
    T = tokens if tokens is not None else max(2 * max(m, n), 16)
    if kind in ("kron", "ho_identity"):
        H_I = damped_gram(_token_matrix(rng, T, n, True, None, 1.0), 0.01)
    else:
        H_I = np.eye(n, dtype=np.float32)
    if kind in ("kron", "hi_identity"):
        H_O = damped_gram(_token_matrix(rng, T, m, True, None, 1.0), 0.01)
    else:
        H_O = np.eye(m, dtype=np.float32)
    return Wstar, H_O, H_I, row_scales(Wstar, bits), bits
