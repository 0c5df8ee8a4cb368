"""Shared test helpers: library factorisations for large inputs and device plumbing."""
import numpy as np


def library_udu(H):
    """U D U^T of H through a library Cholesky (numpy / LAPACK, fp64) of the index-reversed
    matrix: reversal turns the upper factorisation into the usual lower one. Independent of
    the CUDA library under test; used where the oracle's textbook loop is too slow."""
    H = np.asarray(H, dtype=np.float64)
    Hr = H[::-1, ::-1]
    C = np.linalg.cholesky(Hr)
    d = np.diag(C).copy()
    Lr = C / d[None, :]
    L = Lr[::-1, ::-1] - np.eye(H.shape[0])
    return L, (d ** 2)[::-1].copy()


def library_udu_torch(H, device):
    """Same as ``library_udu`` with torch.linalg.cholesky in fp64 on ``device`` (large sizes)."""
    import torch
    Ht = torch.as_tensor(np.ascontiguousarray(H)).to(device=device, dtype=torch.float64)
    Hr = torch.flip(Ht, dims=(0, 1))
    C = torch.linalg.cholesky(Hr)
    del Hr, Ht
    d = torch.diagonal(C).clone()
    C /= d[None, :]
    L = torch.flip(C, dims=(0, 1))
    del C
    L.diagonal().zero_()
    Lf = L.to(torch.float32).cpu().numpy()
    D = torch.flip(d * d, dims=(0,)).cpu().numpy()
    del L, d
    torch.cuda.empty_cache()
    return Lf, D


def cond_estimate(H, device, iters: int = 40, seed: int = 0) -> float:
    """kappa_2(H) of a symmetric positive definite H, estimated in fp64 on ``device``: the
    largest eigenvalue by power iteration, the smallest by inverse iteration through a
    library Cholesky (torch.linalg.cholesky), each as a Rayleigh quotient."""
    import torch
    Ht = torch.as_tensor(np.ascontiguousarray(H)).to(device=device, dtype=torch.float64)
    g = torch.Generator(device=device).manual_seed(seed)
    x = torch.randn(Ht.shape[0], 1, dtype=torch.float64, device=device, generator=g)
    y = x.clone()
    for _ in range(iters):
        x = Ht @ x
        x /= torch.linalg.norm(x)
    lam_max = float((x.T @ Ht @ x).item())
    C = torch.linalg.cholesky(Ht)
    for _ in range(iters):
        y = torch.cholesky_solve(y, C)
        y /= torch.linalg.norm(y)
    lam_min = float((y.T @ Ht @ y).item())
    del Ht, C
    torch.cuda.empty_cache()
    return lam_max / lam_min


def udu_backward_error_rows(H, L, D, rows):
    """For the given rows R: max |((I+L) D (I+L)^T - H)[R, :]| and the scale it is measured
    against, max ((|I+L| D |I+L|^T)[R, :]) (the elementwise backward-error bound of a
    triangular factorisation is a multiple of d eps times the latter), in fp64 on the host."""
    rows = np.asarray(rows)
    d = H.shape[0]
    L64 = np.asarray(L, dtype=np.float64)
    D64 = np.asarray(D, dtype=np.float64)
    UR = L64[rows].copy()
    UR[np.arange(rows.size), rows] += 1.0
    URD = UR * D64[None, :]
    rec = URD @ L64.T + URD            # (U_R D) U^T with U = I + L
    aURD = np.abs(URD)
    scale = aURD @ np.abs(L64).T + aURD
    err = np.abs(rec - np.asarray(H, dtype=np.float64)[rows])
    return float(err.max()), float(scale.max())
