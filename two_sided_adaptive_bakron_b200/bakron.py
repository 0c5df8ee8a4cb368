"""Python binding of libbakron.so (ctypes): argument marshalling only.

The functions named like the C ABI (``bakron_ldl``, ``bakron_round``,
``bakron_round_stochastic``, ``bakron_round_ex``, ``bakron_proxy_loss``, ``bakron_damped_gram``,
``bakron_sketch_b``, ``bakron_rht``, ``bakron_row_scales``, ``bakron_read_status``,
``bakron_status_string`` and the ``*_workspace_bytes`` queries) take torch CUDA tensors, pass
their device pointers and the current CUDA stream to the library and return its status code.
``ldl``, ``round_weights``, ``proxy_loss``, ``damped_gram``, ``sketch_b``, ``rht``,
``row_scales`` and ``solve`` additionally allocate outputs and workspaces with torch and raise
on any error.

Every step of the computation runs in the library's CUDA kernels; there is no CPU path. If
the shared library is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbakron.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "bakron.h")

BAKRON_OK = 0
BAKRON_ERR_INVALID_ARG = -1
BAKRON_ERR_NOT_PD = -2
BAKRON_ERR_CUDA = -3
BAKRON_ERR_TIMEOUT = -4
BAKRON_ERR_WORKSPACE = -5
BAKRON_ERR_NONFINITE = -6
BAKRON_ERR_CAPTURE = -7

_c_size_t, _c_int, _vp = ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p
_SIGNATURES = {
    "bakron_ldl_workspace_bytes": (_c_size_t, [_c_int]),
    "bakron_ldl": (_c_int, [_vp, _c_int, _vp, _vp, _vp, _c_size_t, _vp, _vp]),
    "bakron_round_workspace_bytes": (_c_size_t, [_c_int, _c_int]),
    "bakron_round": (_c_int, [_vp, _c_int, _c_int, _vp, _vp, _vp, _c_int, _vp, _vp, _vp,
                              _c_size_t, _vp, _vp]),
    "bakron_round_stochastic": (_c_int, [_vp, _c_int, _c_int, _vp, _vp, _vp, _c_int,
                                         ctypes.c_uint64, _vp, _vp, _vp, _c_size_t, _vp, _vp]),
    "bakron_round_ex": (_c_int, [_vp, _c_int, _c_int, _vp, _vp, _vp, _c_int, _vp, _c_int, _vp,
                                 _vp, _vp, _c_size_t, _vp, _vp]),
    "bakron_proxy_loss_workspace_bytes": (_c_size_t, [_c_int, _c_int]),
    "bakron_proxy_loss": (_c_int, [_vp, _c_int, _c_int, _vp, _vp, _vp, _vp, _c_size_t, _vp]),
    "bakron_damped_gram_workspace_bytes": (_c_size_t, [_c_int, _c_int]),
    "bakron_damped_gram": (_c_int, [_vp, _c_int, _c_int, ctypes.c_float, _vp, _vp, _c_size_t,
                                    _vp, _vp]),
    "bakron_sketch_b_workspace_bytes": (_c_size_t, [_c_int, _c_int, _c_int]),
    "bakron_sketch_b": (_c_int, [_vp, _c_int, _c_int, _c_int, ctypes.c_float, _vp, _vp, _vp,
                                 _c_size_t, _vp, _vp]),
    "bakron_rht_supported": (_c_int, [_c_int]),
    "bakron_rht_workspace_bytes": (_c_size_t, [_c_int, _c_int]),
    "bakron_rht": (_c_int, [_vp, _c_int, _c_int, ctypes.c_uint64, ctypes.c_uint64, _c_int, _vp,
                            _vp, _c_size_t, _vp]),
    "bakron_row_scales": (_c_int, [_vp, _c_int, _c_int, _c_int, ctypes.c_float, _vp, _vp]),
    "bakron_read_status": (_c_int, [_vp, _vp]),
    "bakron_status_string": (ctypes.c_char_p, [_c_int]),
    "bakron_version": (_c_int, []),
    "bakron_kernel_launches": (ctypes.c_ulonglong, []),
    "bakron_ldl_noalloc": (_c_int, [_vp, _c_int, _vp, _vp, _vp, _vp]),
    "bakron_ldl_noalloc_max_n": (_c_int, []),
    # test hooks (include/bakron_internal.h)
    "bakron_internal_gemm3x_workspace_bytes": (_c_size_t, [_c_int, _c_int, _c_int]),
    "bakron_internal_gemm3x": (_c_int, [_vp, _c_int, _c_int, _c_int, _vp, _c_int, _c_int, _vp,
                                        _c_int, _vp, _c_size_t, _vp, _vp]),
    "bakron_internal_proxy_loss_simt_workspace_bytes": (_c_size_t, [_c_int, _c_int]),
    "bakron_internal_hadamard28": (None, [_vp]),
    "bakron_internal_proxy_loss_simt": (_c_int, [_vp, _c_int, _c_int, _vp, _vp, _vp, _vp,
                                                 _c_size_t, _vp]),
}

_lib: Optional[ctypes.CDLL] = None


class BakronError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {status_string(code)} ({code})")
        self.code = code


def header_functions(path: str = HEADER_PATH) -> list[str]:
    """Names of the functions that a header (default include/bakron.h) declares."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bakron_\w+)\s*\(", text)))


def lib() -> ctypes.CDLL:
    """Loads libbakron.so (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m two_sided_adaptive_bakron_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().bakron_status_string(int(code)).decode()


bakron_status_string = status_string


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check_cuda(t: torch.Tensor, dtype: torch.dtype, shape: tuple, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} of shape {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} contiguous={t.is_contiguous()}")


# ----------------------------------------------------------------------------- C-ABI mirrors
def bakron_ldl_workspace_bytes(n: int) -> int:
    return int(lib().bakron_ldl_workspace_bytes(int(n)))


def bakron_round_workspace_bytes(m: int, n: int) -> int:
    return int(lib().bakron_round_workspace_bytes(int(m), int(n)))


def bakron_proxy_loss_workspace_bytes(m: int, n: int) -> int:
    return int(lib().bakron_proxy_loss_workspace_bytes(int(m), int(n)))


def bakron_ldl(H, L, D, ws, dev_status, stream=None) -> int:
    n = H.shape[0]
    _check_cuda(H, torch.float32, (n, n), "H")
    _check_cuda(L, torch.float32, (n, n), "L")
    _check_cuda(D, torch.float32, (n,), "D")
    return lib().bakron_ldl(_ptr(H), n, _ptr(L), _ptr(D), _ptr(ws), ws.numel() * ws.element_size(),
                            _ptr(dev_status), _stream(stream))


def bakron_round(Wstar, L_O, L_I, scales, bits, codes, W, ws, dev_status, stream=None) -> int:
    m, n = Wstar.shape
    _check_cuda(Wstar, torch.float32, (m, n), "Wstar")
    _check_cuda(L_O, torch.float32, (m, m), "L_O")
    _check_cuda(L_I, torch.float32, (n, n), "L_I")
    _check_cuda(scales, torch.float32, (m,), "scales")
    _check_cuda(codes, torch.int8, (m, n), "codes")
    _check_cuda(W, torch.float32, (m, n), "W")
    return lib().bakron_round(_ptr(Wstar), m, n, _ptr(L_O), _ptr(L_I), _ptr(scales), int(bits),
                              _ptr(codes), _ptr(W), _ptr(ws), ws.numel() * ws.element_size(),
                              _ptr(dev_status), _stream(stream))


def bakron_round_stochastic(Wstar, L_O, L_I, scales, bits, seed, codes, W, ws, dev_status,
                            stream=None) -> int:
    m, n = Wstar.shape
    _check_cuda(Wstar, torch.float32, (m, n), "Wstar")
    _check_cuda(L_O, torch.float32, (m, m), "L_O")
    _check_cuda(L_I, torch.float32, (n, n), "L_I")
    _check_cuda(scales, torch.float32, (m,), "scales")
    _check_cuda(codes, torch.int8, (m, n), "codes")
    _check_cuda(W, torch.float32, (m, n), "W")
    return lib().bakron_round_stochastic(_ptr(Wstar), m, n, _ptr(L_O), _ptr(L_I), _ptr(scales),
                                         int(bits), int(seed) & ((1 << 64) - 1), _ptr(codes),
                                         _ptr(W), _ptr(ws), ws.numel() * ws.element_size(),
                                         _ptr(dev_status), _stream(stream))


def bakron_round_ex(Wstar, L_O, L_I, scales, group_size, codebook, bits, codes, W, ws,
                    dev_status, stream=None) -> int:
    """``scales``: m x G device tensor (G = ceil(n / group_size)); ``codebook``: None or a
    host sequence of 2^bits increasing floats (copied by the call)."""
    m, n = Wstar.shape
    _check_cuda(Wstar, torch.float32, (m, n), "Wstar")
    _check_cuda(L_O, torch.float32, (m, m), "L_O")
    _check_cuda(L_I, torch.float32, (n, n), "L_I")
    gs = min(int(group_size), n)
    _check_cuda(scales, torch.float32, (m, (n + gs - 1) // gs), "scales")
    _check_cuda(codes, torch.int8, (m, n), "codes")
    _check_cuda(W, torch.float32, (m, n), "W")
    cb = None
    if codebook is not None:
        vals = [float(v) for v in codebook]
        cb = (ctypes.c_float * len(vals))(*vals)
    return lib().bakron_round_ex(_ptr(Wstar), m, n, _ptr(L_O), _ptr(L_I), _ptr(scales),
                                 int(group_size), cb, int(bits), _ptr(codes), _ptr(W), _ptr(ws),
                                 ws.numel() * ws.element_size(), _ptr(dev_status),
                                 _stream(stream))


def bakron_proxy_loss(dW, H_O, H_I, loss, ws, stream=None) -> int:
    m, n = dW.shape
    _check_cuda(dW, torch.float32, (m, n), "dW")
    _check_cuda(H_O, torch.float32, (m, m), "H_O")
    _check_cuda(H_I, torch.float32, (n, n), "H_I")
    _check_cuda(loss, torch.float64, (1,), "loss")
    return lib().bakron_proxy_loss(_ptr(dW), m, n, _ptr(H_O), _ptr(H_I), _ptr(loss), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream))


def bakron_damped_gram_workspace_bytes(N: int, d: int) -> int:
    return int(lib().bakron_damped_gram_workspace_bytes(int(N), int(d)))


def bakron_sketch_b_workspace_bytes(S: int, m: int, n: int) -> int:
    return int(lib().bakron_sketch_b_workspace_bytes(int(S), int(m), int(n)))


def bakron_damped_gram(X, damp, H, ws, dev_status, stream=None) -> int:
    N, d = X.shape
    _check_cuda(X, torch.float32, (N, d), "X")
    _check_cuda(H, torch.float32, (d, d), "H")
    return lib().bakron_damped_gram(_ptr(X), N, d, float(damp), _ptr(H), _ptr(ws),
                                    ws.numel() * ws.element_size(), _ptr(dev_status),
                                    _stream(stream))


def bakron_sketch_b(G, damp, H_O, H_I, ws, dev_status, stream=None) -> int:
    S, m, n = G.shape
    _check_cuda(G, torch.float32, (S, m, n), "G")
    _check_cuda(H_O, torch.float32, (m, m), "H_O")
    _check_cuda(H_I, torch.float32, (n, n), "H_I")
    return lib().bakron_sketch_b(_ptr(G), S, m, n, float(damp), _ptr(H_O), _ptr(H_I), _ptr(ws),
                                 ws.numel() * ws.element_size(), _ptr(dev_status),
                                 _stream(stream))


def bakron_rht_supported(d: int) -> bool:
    return bool(lib().bakron_rht_supported(int(d)))


def bakron_rht_workspace_bytes(rows: int, cols: int) -> int:
    return int(lib().bakron_rht_workspace_bytes(int(rows), int(cols)))


def bakron_rht(X, seed_rows, seed_cols, inverse, Y, ws, stream=None) -> int:
    r, c = X.shape
    _check_cuda(X, torch.float32, (r, c), "X")
    _check_cuda(Y, torch.float32, (r, c), "Y")
    m64 = (1 << 64) - 1
    return lib().bakron_rht(_ptr(X), r, c, int(seed_rows) & m64, int(seed_cols) & m64,
                            int(bool(inverse)), _ptr(Y), _ptr(ws), ws.numel() * ws.element_size(),
                            _stream(stream))


def bakron_row_scales(W, group_size, divisor, scales, stream=None) -> int:
    m, n = W.shape
    _check_cuda(W, torch.float32, (m, n), "W")
    g = min(int(group_size), n)
    _check_cuda(scales, torch.float32, (m, (n + g - 1) // g), "scales")
    return lib().bakron_row_scales(_ptr(W), m, n, int(group_size), float(divisor), _ptr(scales),
                                   _stream(stream))


def internal_hadamard28():
    """The order-28 Hadamard matrix the library's transform uses (host construction)."""
    import numpy as np
    buf = (ctypes.c_byte * 784)()
    lib().bakron_internal_hadamard28(buf)
    return np.frombuffer(bytes(buf), dtype=np.int8).reshape(28, 28).copy()


def bakron_ldl_noalloc(H, L, D, dev_status, stream=None) -> int:
    """bakron_ldl with the library's own fixed scratch (no workspace argument)."""
    n = H.shape[0]
    _check_cuda(H, torch.float32, (n, n), "H")
    _check_cuda(L, torch.float32, (n, n), "L")
    _check_cuda(D, torch.float32, (n,), "D")
    return lib().bakron_ldl_noalloc(_ptr(H), n, _ptr(L), _ptr(D), _ptr(dev_status),
                                    _stream(stream))


def bakron_ldl_noalloc_max_n() -> int:
    return int(lib().bakron_ldl_noalloc_max_n())


def bakron_read_status(dev_status, stream=None) -> int:
    return int(lib().bakron_read_status(_ptr(dev_status), _stream(stream)))


def bakron_kernel_launches() -> int:
    return int(lib().bakron_kernel_launches())


def bakron_version() -> int:
    return int(lib().bakron_version())


def internal_gemm3x(A: torch.Tensor, B: torch.Tensor, stream=None) -> torch.Tensor:
    """C = A B^T through the 3xTF32 tensor-core engine (test hook)."""
    M, K = A.shape
    N = B.shape[0]
    C = torch.empty((M, N), dtype=torch.float32, device=A.device)
    ws = workspace(int(lib().bakron_internal_gemm3x_workspace_bytes(M, N, K)), A.device)
    st = new_status(A.device)
    _raise(lib().bakron_internal_gemm3x(_ptr(A), M, K, A.stride(0), _ptr(B), N, B.stride(0),
                                        _ptr(C), N, _ptr(ws), ws.numel(), _ptr(st),
                                        _stream(stream)), "bakron_internal_gemm3x")
    _raise(bakron_read_status(st, stream), "bakron_internal_gemm3x (device)")
    return C


def internal_proxy_loss_simt(dW, H_O, H_I, stream=None) -> torch.Tensor:
    """The CUDA-core proxy loss (test hook, cross-check of bakron_proxy_loss)."""
    m, n = dW.shape
    loss = torch.empty((1,), dtype=torch.float64, device=dW.device)
    ws = workspace(int(lib().bakron_internal_proxy_loss_simt_workspace_bytes(m, n)), dW.device)
    _raise(lib().bakron_internal_proxy_loss_simt(_ptr(dW), m, n, _ptr(H_O), _ptr(H_I),
                                                 _ptr(loss), _ptr(ws), ws.numel(),
                                                 _stream(stream)), "proxy_loss_simt")
    return loss


# ----------------------------------------------------------------------------- conveniences
def workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte aligned byte buffer (torch's caching allocator aligns to 512 bytes)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def new_status(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def _raise(code: int, where: str):
    if code != BAKRON_OK:
        raise BakronError(code, where)


def ldl(H: torch.Tensor, stream=None, check: bool = True):
    """(L, D) with H = (I + L) diag(D) (I + L)^T, L strictly upper."""
    n = H.shape[0]
    L = torch.empty((n, n), dtype=torch.float32, device=H.device)
    D = torch.empty((n,), dtype=torch.float32, device=H.device)
    ws = workspace(bakron_ldl_workspace_bytes(n), H.device)
    st = new_status(H.device)
    _raise(bakron_ldl(H, L, D, ws, st, stream), "bakron_ldl")
    if check:
        _raise(bakron_read_status(st, stream), "bakron_ldl (device)")
    return L, D


def round_weights(Wstar, L_O, L_I, scales, bits, stream=None, check: bool = True, seed=None,
                  group_size=None, codebook=None):
    """(codes int8, W fp32) of the BaKron solve; a seed selects stochastic Q, a group size
    (with m x G scales) and/or a host codebook select the base quantizer of bakron_round_ex."""
    m, n = Wstar.shape
    codes = torch.empty((m, n), dtype=torch.int8, device=Wstar.device)
    W = torch.empty((m, n), dtype=torch.float32, device=Wstar.device)
    ws = workspace(bakron_round_workspace_bytes(m, n), Wstar.device)
    st = new_status(Wstar.device)
    if group_size is not None or codebook is not None:
        if seed is not None:
            raise ValueError("stochastic Q takes the per-row integer grid")
        _raise(bakron_round_ex(Wstar, L_O, L_I, scales, n if group_size is None else group_size,
                               codebook, bits, codes, W, ws, st, stream), "bakron_round_ex")
    elif seed is None:
        _raise(bakron_round(Wstar, L_O, L_I, scales, bits, codes, W, ws, st, stream),
               "bakron_round")
    else:
        _raise(bakron_round_stochastic(Wstar, L_O, L_I, scales, bits, seed, codes, W, ws, st,
                                       stream), "bakron_round_stochastic")
    if check:
        _raise(bakron_read_status(st, stream), "bakron_round (device)")
    return codes, W


def damped_gram(X, damp: float = 0.01, stream=None, check: bool = True) -> torch.Tensor:
    """X^T X / N + damp * mean(diag) * I for samples X (N x d) on the device."""
    N, d = X.shape
    H = torch.empty((d, d), dtype=torch.float32, device=X.device)
    ws = workspace(bakron_damped_gram_workspace_bytes(N, d), X.device)
    st = new_status(X.device)
    _raise(bakron_damped_gram(X, damp, H, ws, st, stream), "bakron_damped_gram")
    if check:
        _raise(bakron_read_status(st, stream), "bakron_damped_gram (device)")
    return H


def sketch_b(G, damp: float = 0.01, stream=None, check: bool = True):
    """(H_O, H_I) of Sketch B from per-sequence gradients G (S x m x n) on the device."""
    S, m, n = G.shape
    H_O = torch.empty((m, m), dtype=torch.float32, device=G.device)
    H_I = torch.empty((n, n), dtype=torch.float32, device=G.device)
    ws = workspace(bakron_sketch_b_workspace_bytes(S, m, n), G.device)
    st = new_status(G.device)
    _raise(bakron_sketch_b(G, damp, H_O, H_I, ws, st, stream), "bakron_sketch_b")
    if check:
        _raise(bakron_read_status(st, stream), "bakron_sketch_b (device)")
    return H_O, H_I


def rht(X, seed_rows: int, seed_cols: int, inverse: bool = False, stream=None) -> torch.Tensor:
    """T_rows X T_cols^T (inverse: T_rows^T X T_cols) on the device (a new tensor)."""
    Y = torch.empty_like(X)
    ws = workspace(bakron_rht_workspace_bytes(*X.shape), X.device)
    _raise(bakron_rht(X, seed_rows, seed_cols, inverse, Y, ws, stream), "bakron_rht")
    return Y


def row_scales(W, divisor: float, group_size=None, stream=None) -> torch.Tensor:
    """max |W| over each row (and group of columns) / divisor, on the device."""
    m, n = W.shape
    g = n if group_size is None else min(int(group_size), n)
    out = torch.empty((m, (n + g - 1) // g), dtype=torch.float32, device=W.device)
    _raise(bakron_row_scales(W, g, divisor, out, stream), "bakron_row_scales")
    return out if group_size is not None else out.view(m)


def proxy_loss(dW, H_O, H_I, stream=None) -> torch.Tensor:
    """tr(H_O dW H_I dW^T) as a one-element float64 CUDA tensor."""
    m, n = dW.shape
    loss = torch.empty((1,), dtype=torch.float64, device=dW.device)
    ws = workspace(bakron_proxy_loss_workspace_bytes(m, n), dW.device)
    _raise(bakron_proxy_loss(dW, H_O, H_I, loss, ws, stream), "bakron_proxy_loss")
    return loss


class Solver:
    """Reusable buffers for the whole path: ldl(H_O), ldl(H_I), round, proxy loss.

    The round workspace keeps E = W* - W at its start (see bakron.h), which is the dW handed
    to the proxy loss.
    """

    def __init__(self, m: int, n: int, device="cuda"):
        self.m, self.n, self.device = m, n, torch.device(device)
        f32 = dict(dtype=torch.float32, device=self.device)
        self.L_O = torch.empty((m, m), **f32)
        self.D_O = torch.empty((m,), **f32)
        self.L_I = torch.empty((n, n), **f32)
        self.D_I = torch.empty((n,), **f32)
        self.codes = torch.empty((m, n), dtype=torch.int8, device=self.device)
        self.W = torch.empty((m, n), **f32)
        self.loss = torch.empty((1,), dtype=torch.float64, device=self.device)
        self.ws_round = workspace(bakron_round_workspace_bytes(m, n), self.device)
        self.ws_O = workspace(bakron_ldl_workspace_bytes(m), self.device)
        self.ws = workspace(max(bakron_ldl_workspace_bytes(n),
                                bakron_proxy_loss_workspace_bytes(m, n)), self.device)
        self.E = self.ws_round[: 4 * m * n].view(torch.float32).view(m, n)
        self._rot = None     # incoherence buffers, made on first use
        self.status = new_status(self.device)
        # the two factorisations are independent: ldl(H_O) runs on a side stream while
        # ldl(H_I) runs on the caller's stream
        self.side = torch.cuda.Stream(device=self.device)
        self._fork = torch.cuda.Event()
        self._join = torch.cuda.Event()

    def _rotated(self):
        if self._rot is None:
            m, n, dev = self.m, self.n, self.device
            f32 = dict(dtype=torch.float32, device=dev)
            self._rot = dict(W=torch.empty((m, n), **f32), HO=torch.empty((m, m), **f32),
                             HI=torch.empty((n, n), **f32), s=torch.empty((m, 1), **f32),
                             W_orig=torch.empty((m, n), **f32),
                             ws=workspace(max(bakron_rht_workspace_bytes(m, n),
                                              bakron_rht_workspace_bytes(m, m),
                                              bakron_rht_workspace_bytes(n, n)), dev))
        return self._rot

    def run(self, Wstar, H_O, H_I, scales, bits, stream=None, with_loss=True, timing=None,
            seed=None, group_size=None, codebook=None, incoherence=None):
        """Enqueues the whole path (reads: self.codes, self.W, self.E, self.loss); a seed
        selects stochastic Q for the round, a group size (with m x G scales) and/or a host
        codebook the base quantizer of bakron_round_ex.

        incoherence=(seed_o, seed_i) runs the path on the rotated layer (bakron_rht):
        W~ = T_m W* T_n^T, H_O~ = T_m H_O T_m^T, H_I~ = T_n H_I T_n^T, per-row grid steps of
        W~ (``scales`` is then ignored), and writes self.W_orig = T_m^T W~_q T_n. self.codes,
        self.W and self.E stay in the rotated basis, where the proxy loss is the same.

        timing: optional {name: (start_event, end_event)} for any of "ldl_O", "ldl_I", "round",
        "loss"; each pair is recorded around its call on the stream that runs it.
        """
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        timing = timing or {}
        if incoherence is not None:
            if group_size is not None or codebook is not None:
                raise ValueError("incoherence processing takes per-row integer-grid steps")
            so, si = incoherence
            R = self._rotated()
            ev = timing.get("rotate")
            if ev is not None:
                ev[0].record(stream)
            for X, Y, a, b in ((Wstar, R["W"], so, si), (H_O, R["HO"], so, so),
                               (H_I, R["HI"], si, si)):
                _raise(bakron_rht(X, a, b, False, Y, R["ws"], stream), "bakron_rht")
            _raise(bakron_row_scales(R["W"], self.n, (1 << (bits - 1)) - 0.5, R["s"], stream),
                   "bakron_row_scales")
            if ev is not None:
                ev[1].record(stream)
            Wstar, H_O, H_I, scales = R["W"], R["HO"], R["HI"], R["s"].view(self.m)

        def call(name, st, fn, *a):
            ev = timing.get(name)
            if ev is not None:
                ev[0].record(st)
            _raise(fn(*a, st), "bakron " + name)
            if ev is not None:
                ev[1].record(st)

        self._fork.record(stream)
        self.side.wait_event(self._fork)
        call("ldl_O", self.side, bakron_ldl, H_O, self.L_O, self.D_O, self.ws_O, self.status)
        call("ldl_I", stream, bakron_ldl, H_I, self.L_I, self.D_I, self.ws, self.status)
        self._join.record(self.side)
        stream.wait_event(self._join)
        if group_size is not None or codebook is not None:
            call("round", stream, bakron_round_ex, Wstar, self.L_O, self.L_I, scales,
                 self.n if group_size is None else group_size, codebook, bits, self.codes,
                 self.W, self.ws_round, self.status)
        elif seed is None:
            call("round", stream, bakron_round, Wstar, self.L_O, self.L_I, scales, bits,
                 self.codes, self.W, self.ws_round, self.status)
        else:
            call("round", stream, bakron_round_stochastic, Wstar, self.L_O, self.L_I, scales,
                 bits, seed, self.codes, self.W, self.ws_round, self.status)
        if with_loss:
            call("loss", stream, bakron_proxy_loss, self.E, H_O, H_I, self.loss, self.ws)
        if incoherence is not None:
            R = self._rotated()
            ev = timing.get("unrotate")
            if ev is not None:
                ev[0].record(stream)
            _raise(bakron_rht(self.W, so, si, True, R["W_orig"], R["ws"], stream), "bakron_rht")
            if ev is not None:
                ev[1].record(stream)
            self.W_orig = R["W_orig"]

    def check(self, stream=None):
        _raise(bakron_read_status(self.status, stream), "bakron (device)")


def solve(Wstar, H_O, H_I, scales, bits, stream=None, seed=None):
    """Whole path on device tensors: returns (codes, W, loss, (L_O, D_O), (L_I, D_I)); a seed
    selects stochastic Q."""
    s = Solver(Wstar.shape[0], Wstar.shape[1], Wstar.device)
    s.run(Wstar, H_O, H_I, scales, bits, stream, seed=seed)
    s.check(stream)
    return s.codes, s.W, s.loss, (s.L_O, s.D_O), (s.L_I, s.D_I)
