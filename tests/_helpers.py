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
