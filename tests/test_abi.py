"""CPU checks of the C ABI: the library builds, loads without a GPU and exports every function
declared in include/bakron.h; host-side helpers behave."""
import ctypes

import pytest

from two_sided_adaptive_bakron_b200 import build as B


@pytest.fixture(scope="module")
def libpath():
    return B.build()


def test_library_exports_every_header_function(libpath):
    from two_sided_adaptive_bakron_b200 import bakron
    names = bakron.header_functions()
    assert {"bakron_ldl", "bakron_round", "bakron_proxy_loss", "bakron_read_status",
            "bakron_status_string", "bakron_ldl_workspace_bytes",
            "bakron_round_workspace_bytes", "bakron_proxy_loss_workspace_bytes"} <= set(names)
    lib = ctypes.CDLL(libpath)
    names += bakron.header_functions(bakron.HEADER_PATH.replace("bakron.h", "bakron_internal.h"))
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_host_side_queries_without_gpu(libpath):
    from two_sided_adaptive_bakron_b200 import bakron
    assert bakron.bakron_version() >= 100
    assert bakron.status_string(0) == "ok"
    assert "timed out" in bakron.status_string(-4)
    assert "capture" in bakron.status_string(bakron.BAKRON_ERR_CAPTURE)
    # every status the header declares has its own message
    import re
    with open(bakron.HEADER_PATH) as f:
        codes = [int(v) for v in re.findall(r"BAKRON_ERR_\w+ = (-\d+)", f.read())]
    assert len(codes) >= 7
    assert len({bakron.status_string(c) for c in codes}) == len(codes)
    assert all(bakron.status_string(c) != "unknown status" for c in codes)
    assert bakron.bakron_round_workspace_bytes(0, 5) == 0
    m, n = 100, 37
    assert bakron.bakron_round_workspace_bytes(m, n) >= 2 * 4 * m * n
    assert bakron.bakron_ldl_workspace_bytes(1000) > 0
    assert bakron.bakron_proxy_loss_workspace_bytes(m, n) >= 4 * m * n


def test_invalid_arguments_rejected_on_host(libpath):
    lib = ctypes.CDLL(libpath)
    lib.bakron_round.restype = ctypes.c_int
    vp = ctypes.c_void_p
    lib.bakron_round.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, vp, vp, ctypes.c_int, vp,
                                 vp, vp, ctypes.c_size_t, vp, vp]
    fake = vp(0x1000)
    # bits out of range
    assert lib.bakron_round(fake, 4, 4, fake, fake, fake, 1, fake, fake, fake, 1 << 20, fake,
                            None) == -1
    # empty matrix
    assert lib.bakron_round(fake, 0, 4, fake, fake, fake, 2, fake, fake, fake, 1 << 20, fake,
                            None) == -1
    # workspace too small / misaligned
    assert lib.bakron_round(fake, 4, 4, fake, fake, fake, 2, fake, fake, vp(0x1000), 16, fake,
                            None) == -5
    assert lib.bakron_round(fake, 4, 4, fake, fake, fake, 2, fake, fake, vp(0x1001), 1 << 20,
                            fake, None) == -5
    lib.bakron_ldl.restype = ctypes.c_int
    lib.bakron_ldl.argtypes = [vp, ctypes.c_int, vp, vp, vp, ctypes.c_size_t, vp, vp]
    assert lib.bakron_ldl(fake, 0, fake, fake, fake, 1 << 20, fake, None) == -1


def test_new_entry_points_reject_bad_arguments_on_host(libpath):
    """Argument checks of the stochastic, quantizer and Kronecker-factor entry points return
    before any device work (no GPU needed)."""
    lib = ctypes.CDLL(libpath)
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fake, big = vp(0x1000), 1 << 30
    lib.bakron_round_stochastic.restype = ci
    lib.bakron_round_stochastic.argtypes = [vp, ci, ci, vp, vp, vp, ci, ctypes.c_uint64, vp, vp,
                                            vp, ctypes.c_size_t, vp, vp]
    assert lib.bakron_round_stochastic(fake, 4, 4, fake, fake, fake, 9, 1, fake, fake, fake, big,
                                       fake, None) == -1
    lib.bakron_round_ex.restype = ci
    lib.bakron_round_ex.argtypes = [vp, ci, ci, vp, vp, vp, ci, vp, ci, vp, vp, vp,
                                    ctypes.c_size_t, vp, vp]

    def ex(n, group, book, bits, ws_bytes=big):
        cb = None if book is None else (cf * len(book))(*book)
        return lib.bakron_round_ex(fake, 8, n, fake, fake, fake, group, cb, bits, fake, fake,
                                   fake, ws_bytes, fake, None)
    assert ex(64, 48, None, 3) == -1                       # group not a multiple of 32
    assert ex(64, 0, None, 3) == -1
    assert ex(64, 32, [0.0, 2.0, 1.0, 3.0], 2) == -1       # not increasing
    assert ex(64, 32, [0.0, 0.0, 1.0, 3.0], 2) == -1       # not strictly increasing
    assert ex(64, 32, [0.0, 1.0, float("nan"), 3.0], 2) == -1
    assert ex(64, 32, [float(k) for k in range(32)], 5) == -1   # more than 16 entries
    assert ex(64, 32, None, 9) == -1
    assert ex(64, 32, [0.0, 1.0], 1, ws_bytes=16) == -5    # valid: then the tiny workspace fails
    lib.bakron_damped_gram.restype = ci
    lib.bakron_damped_gram.argtypes = [vp, ci, ci, cf, vp, vp, ctypes.c_size_t, vp, vp]
    assert lib.bakron_damped_gram(fake, 0, 4, 0.01, fake, fake, big, fake, None) == -1
    assert lib.bakron_damped_gram(fake, 4, 4, -0.5, fake, fake, big, fake, None) == -1
    assert lib.bakron_damped_gram(fake, 4, 70000, 0.01, fake, fake, big, fake, None) == -1
    assert lib.bakron_damped_gram(fake, 4, 4, 0.01, fake, vp(0x1001), big, fake, None) == -5
    lib.bakron_sketch_b.restype = ci
    lib.bakron_sketch_b.argtypes = [vp, ci, ci, ci, cf, vp, vp, vp, ctypes.c_size_t, vp, vp]
    assert lib.bakron_sketch_b(fake, 0, 4, 4, 0.01, fake, fake, fake, big, fake, None) == -1
    assert lib.bakron_sketch_b(fake, 2, 4, 4, 0.01, fake, fake, fake, 16, fake, None) == -5
    lib.bakron_damped_gram_workspace_bytes.restype = ctypes.c_size_t
    lib.bakron_damped_gram_workspace_bytes.argtypes = [ci, ci]
    assert lib.bakron_damped_gram_workspace_bytes(1000, 300) >= 2 * 300 * 1000 * 4


def test_library_hadamard28_equals_the_oracle(libpath):
    """The library builds H_28 on the host from its own GF(27) arithmetic; it must be the
    oracle's matrix (checked here, without a GPU)."""
    import numpy as np

    import oracle
    from two_sided_adaptive_bakron_b200 import bakron
    np.testing.assert_array_equal(bakron.internal_hadamard28().astype(np.float64),
                                  oracle.hadamard28())
    assert all(bakron.bakron_rht_supported(d) for d in (1, 2, 28, 56, 4096, 14336, 28672, 32768))
    assert not any(bakron.bakron_rht_supported(d) for d in (0, 3, 12, 20, 84, 65536, 57344))


def test_rht_rejects_bad_arguments_on_host(libpath):
    lib = ctypes.CDLL(libpath)
    vp, ci = ctypes.c_void_p, ctypes.c_int
    lib.bakron_rht.restype = ci
    lib.bakron_rht.argtypes = [vp, ci, ci, ctypes.c_uint64, ctypes.c_uint64, ci, vp, vp,
                               ctypes.c_size_t, vp]
    fake = vp(0x1000)
    assert lib.bakron_rht(fake, 12, 28, 1, 2, 0, fake, fake, 1 << 30, None) == -1
    assert lib.bakron_rht(fake, 28, 28, 1, 2, 2, fake, fake, 1 << 30, None) == -1
    assert lib.bakron_rht(fake, 28, 28, 1, 2, 0, fake, fake, 16, None) == -5
    lib.bakron_row_scales.restype = ci
    lib.bakron_row_scales.argtypes = [vp, ci, ci, ci, ctypes.c_float, vp, vp]
    assert lib.bakron_row_scales(fake, 4, 4, 4, 0.0, fake, None) == -1


def test_missing_library_fails_loudly(monkeypatch):
    """There is no CPU fallback: without the built library every call raises."""
    from two_sided_adaptive_bakron_b200 import bakron
    monkeypatch.setattr(bakron, "_lib", None)
    monkeypatch.setattr(bakron, "LIB_PATH", "/nonexistent/libbakron.so")
    with pytest.raises(RuntimeError, match="missing"):
        bakron.bakron_version()
    with pytest.raises(RuntimeError, match="missing"):
        bakron.bakron_round_workspace_bytes(8, 8)
