"""Runs one entry point of the library on a synthetic input, for timing and profiling.

    python -m two_sided_adaptive_bakron_b200.kernel_bench --op OP [--workload NAME]
                                                          [--d D] [--k K] [--iters I]

OP is one of
  ldl       bakron_ldl of the workload's H_I (or of a damped Gram of size --d)
  round     bakron_round of the workload with library-made factors
  loss      bakron_proxy_loss of a random residual with the workload's H_O, H_I
  gram      bakron_damped_gram of a --k x --d Gaussian sample matrix
  sketch_b  bakron_sketch_b of --k Gaussian gradients of the workload's shape (<= 4 GiB)
  rht       bakron_rht of a Gaussian matrix of the workload's shape, then its inverse
The call is made --iters times (the first is a warm-up) and the mean time of the others is
printed, from CUDA events on the launching stream. Inputs come from the seeded generators of
``workloads``; everything runs through the ctypes binding of the C ABI.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main(argv=None) -> int:
    import torch

    from two_sided_adaptive_bakron_b200 import bakron as bk
    from two_sided_adaptive_bakron_b200.workloads import WORKLOADS, make_workload, random_problem

    ap = argparse.ArgumentParser()
    ap.add_argument("--op", required=True,
                    choices=["ldl", "round", "loss", "gram", "sketch_b", "rht"])
    ap.add_argument("--workload", default="attn_4096", choices=sorted(WORKLOADS))
    ap.add_argument("--d", type=int, default=0)
    ap.add_argument("--k", type=int, default=4096)
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args(argv)
    dev = torch.device("cuda")
    d = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    wl = WORKLOADS[a.workload]
    rng = np.random.default_rng(7)

    if a.op in ("ldl", "round", "loss"):
        if a.op == "ldl" and a.d:
            _, H, _, _, _ = random_problem(a.d, 1, 2, 7)
            Ws = HO = None
            HI = H
        else:
            Ws, HO, HI, s, bits = make_workload(wl, device="cuda")
    if a.op == "ldl":
        H = d(HI)
        fn = lambda: bk.ldl(H)
    elif a.op == "round":
        LO, _ = bk.ldl(d(HO))
        LI, _ = bk.ldl(d(HI))
        dW, ds = d(Ws), d(s)
        fn = lambda: bk.round_weights(dW, LO, LI, ds, bits)
    elif a.op == "loss":
        dW = d((rng.standard_normal(Ws.shape) * 0.01).astype(np.float32))
        dHO, dHI = d(HO), d(HI)
        fn = lambda: bk.proxy_loss(dW, dHO, dHI)
    elif a.op == "gram":
        X = d(rng.standard_normal((a.k, a.d or wl.n)).astype(np.float32))
        fn = lambda: bk.damped_gram(X, wl.damp)
    elif a.op == "sketch_b":
        if a.k * wl.m * wl.n * 4 > (4 << 30):
            raise SystemExit("sketch_b: --k gradients of the workload's shape exceed 4 GiB")
        G = torch.randn((a.k, wl.m, wl.n), generator=torch.Generator(device=dev).manual_seed(7),
                        device=dev)
        fn = lambda: bk.sketch_b(G, wl.damp)
    else:
        X = d(rng.standard_normal((wl.m, wl.n)).astype(np.float32))
        fn = lambda: bk.rht(bk.rht(X, 11, 12), 11, 12, inverse=True)

    times = []
    for i in range(max(1, a.iters)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        if i > 0 or a.iters == 1:
            times.append(e0.elapsed_time(e1))
    print(f"{a.op} {a.workload if not (a.op in ('ldl', 'gram') and a.d) else a.d}: "
          f"{sum(times) / len(times):.3f} ms (mean of {len(times)})", flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
