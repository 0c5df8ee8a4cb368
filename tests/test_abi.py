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
