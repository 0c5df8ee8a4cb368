"""GPU check of bakron_ldl_noalloc, the factorisation for callers that cannot allocate device
memory (its scratch is a fixed array inside the library instead of a caller workspace).

It must give the same factors as bakron_ldl with a caller workspace, on two calls in a row
(the second call reuses the array the first one left behind), and reject sizes above its
limit. This file is collected last so that a stop-at-first-failure run has already run every
other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from two_sided_adaptive_bakron_b200 import build
    build.build()
    from two_sided_adaptive_bakron_b200 import bakron
    return bakron


def _factor_noalloc(bk, H):
    n = H.shape[0]
    L = torch.full((n, n), float("nan"), device="cuda")
    D = torch.full((n,), float("nan"), device="cuda")
    st = bk.new_status("cuda")
    assert bk.bakron_ldl_noalloc(H, L, D, st) == bk.BAKRON_OK
    assert bk.bakron_read_status(st) == bk.BAKRON_OK
    return L.cpu().numpy(), D.cpu().numpy()


@pytest.mark.parametrize("n,seed", [(300, 1), (2048, 2)])
def test_noalloc_ldl_matches_workspace_ldl_twice(bk, n, seed):
    from two_sided_adaptive_bakron_b200.workloads import random_problem
    _, H_np, _, _, _ = random_problem(n, 3, 2, seed)
    H = torch.from_numpy(H_np).cuda()
    L_ref, D_ref = bk.ldl(H)
    L_ref, D_ref = L_ref.cpu().numpy(), D_ref.cpu().numpy()
    for _ in range(2):
        L, D = _factor_noalloc(bk, H)
        # same kernels, same inputs: the ldl tests' tolerance, met here with equality
        np.testing.assert_allclose(L, L_ref, rtol=0, atol=1e-6 * max(1.0, np.abs(L_ref).max()))
        np.testing.assert_allclose(D, D_ref, rtol=1e-6)
        assert np.array_equal(L, L_ref) and np.array_equal(D, D_ref)


def test_noalloc_ldl_rejects_too_large(bk):
    n = bk.bakron_ldl_noalloc_max_n() + 1
    H = torch.eye(n, device="cuda")
    L = torch.empty((n, n), device="cuda")
    D = torch.empty((n,), device="cuda")
    st = bk.new_status("cuda")
    assert bk.bakron_ldl_noalloc(H, L, D, st) == bk.BAKRON_ERR_INVALID_ARG


def test_noalloc_first_call_under_capture_is_refused(bk):
    """The first call in a fresh process, made while its stream captures a CUDA graph, must
    not look up the scratch address (that may load the module): it returns BAKRON_ERR_CAPTURE
    and leaves the capture intact; the same call after the capture works."""
    import os
    import subprocess
    import sys
    code = r"""
import numpy as np, torch
from two_sided_adaptive_bakron_b200 import bakron as bk
from two_sided_adaptive_bakron_b200.workloads import random_problem
_, H_np, _, _, _ = random_problem(64, 3, 2, 5)
H = torch.from_numpy(H_np).cuda()
L = torch.empty((64, 64), device='cuda'); D = torch.empty((64,), device='cuda')
st = bk.new_status('cuda')
bk.lib()
s = torch.cuda.Stream()
torch.cuda.synchronize()
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g, stream=s):
    rc = bk.bakron_ldl_noalloc(H, L, D, st, stream=s)
print('CAPTURED', rc)
rc2 = bk.bakron_ldl_noalloc(H, L, D, st)
print('AFTER', rc2, bk.bakron_read_status(st))
Lr, Dr = bk.ldl(H)
print('SAME', bool(torch.equal(L, Lr) and torch.equal(D, Dr)))
"""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    assert f"CAPTURED {bk.BAKRON_ERR_CAPTURE}" in r.stdout, r.stdout
    assert "AFTER 0 0" in r.stdout and "SAME True" in r.stdout, r.stdout
