"""Benchmark of the BaKron solve path on synthetic LLM-layer workloads.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
                    [--rounding nearest|stochastic] [--hessian]
                    [--group-size G] [--codebook normal] [--incoherence]

One step = the whole path on one layer with inputs resident in HBM:
    bakron_ldl(H_O), bakron_ldl(H_I), bakron_round(W*, L_O, L_I, scales, bits),
    bakron_proxy_loss(W* - W, H_O, H_I).
--hessian adds the two damped Kronecker factors to the step: bakron_damped_gram builds H_I from
the layer's token matrix X and H_O from its gradient rows G (resident in HBM) before the solve.
--group-size G / --codebook normal time bakron_round_ex: one grid step per row and group of G
columns (max |W*| over the group / the grid's top), and/or the 2^bits-entry codebook of normal
quantiles (k + 1/2) / 2^bits scaled to [-1, 1].
--incoherence adds the two-sided randomised Hadamard transform (bakron_rht) of W*, H_O and
H_I, the grid steps of the rotated W* (bakron_row_scales) and the inverse transform of the
rounded weights to the step.
--rounding stochastic times bakron_round_stochastic (stochastic Q, a fixed seed per step) in
place of bakron_round. Metric: quantized weights per second, m*n / step time (whole job: summed over replicas, one
independent layer per GPU, no collective on the data path; timed as the max over ranks).

--impl reference times the fp64 CPU oracle (the deliberately slow reference) on a bounded
sample of the same workload: its O(mn(m+n)) row sweep of the rounding rule on the leading r
full-width rows of the layer (W*[:r, :], L_O[:r, :r], L_I), with every host thread available
to numpy; weights/s = r*n / t. The same sample is the main line's cpu_baseline.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "BaKron solver quantized weights/s (m·n/s) and % of B200 tensor roofline"
UNIT = "weights/s"
DEFAULT_WORKLOAD = "down_4096x14336"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """SM clock and clock-event reasons sampled while the timed region runs (reads only).

    NVML is read every 10 ms from a thread; without NVML, nvidia-smi samples every 100 ms,
    and the timed region starts only after its first line, so a short region still gets
    samples. Any failure leaves the summary empty; it never stops the benchmark.
    """

    PERIOD_S = 0.01
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown", 0x8),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap", 0x4))

    def __init__(self, index: int):
        self.index = index
        self.source = None
        self.proc = None
        self.lines: list[str] = []
        self.samples: list[tuple[float, int]] = []   # NVML: (SM MHz, reason bits)
        self.max_mhz = None
        self.mark = 0

    def __enter__(self):
        if not self._start_nvml():
            self._start_smi()
        return self

    def _start_nvml(self) -> bool:
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)   # both reads work here
            reasons(h)
        except Exception:
            return False
        self.nvml, self.bits = pynvml, {nm: int(getattr(pynvml, attr, dflt))
                                        for nm, attr, dflt in self.REASONS}
        self.stop = threading.Event()

        def loop():
            while not self.stop.is_set():
                try:
                    self.samples.append((float(pynvml.nvmlDeviceGetClockInfo(
                        h, pynvml.NVML_CLOCK_SM)), int(reasons(h))))
                except Exception:
                    pass
                self.stop.wait(self.PERIOD_S)

        self.t = threading.Thread(target=loop, daemon=True)
        self.t.start()
        self.source = "nvml"
        return True

    def _start_smi(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.source = "nvidia-smi"
        self.first = threading.Event()
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()
        self.first.wait(3.0)            # the tool is up; samples from here on
        self.mark = len(self.lines)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())
            self.first.set()

    def __exit__(self, *exc):
        if self.source == "nvml":
            self.stop.set()
            self.t.join(timeout=1.0)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], self.max_mhz, set()
        if self.source == "nvml":
            for mhz, r in self.samples:
                sm.append(mhz)
                reasons.update(nm for nm, bit in self.bits.items() if r & bit)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines[self.mark:]:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def normal_codebook(bits: int):
    """2^bits normal quantiles at (k + 1/2) / 2^bits, scaled to [-1, 1] (fp32)."""
    import numpy as np
    from statistics import NormalDist
    K = 1 << bits
    q = np.array([NormalDist().inv_cdf((k + 0.5) / K) for k in range(K)])
    return (q / np.abs(q).max()).astype(np.float32)


def max_over_ranks(x: float, device) -> float:
    """The maximum of x over all ranks, returned on every rank (x itself without a process
    group): a multi-GPU time is the slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world: int, m: int, n: int, ms_per_step: float) -> float:
    """Weights per second of the whole job: each of the `world` replicas rounds its own m x n
    layer per step, and the step takes the slowest rank's time."""
    return world * m * n / (ms_per_step * 1e-3)


def _gram_device(wl):
    """Where the input generator forms the large Gram products: the GPU when there is one
    (the inputs only; the oracle itself runs on the host)."""
    import torch
    return "cuda" if wl.m * wl.n > (1 << 22) and torch.cuda.is_available() else None


def _lapack_udu(H):
    """Strictly upper L of H = (I + L) D (I + L)^T via LAPACK's Cholesky of the index-reversed
    matrix (numpy, fp64): the factors the CPU row sweep consumes, formed outside its timing."""
    import numpy as np
    Hr = np.asarray(H, dtype=np.float64)[::-1, ::-1]
    C = np.linalg.cholesky(Hr)
    L = (C / np.diag(C)[None, :])[::-1, ::-1].copy()
    L[np.diag_indices_from(L)] = 0.0
    return L


def cpu_info():
    """Host threads this process may use and the CPU model."""
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            model = next((ln.split(":", 1)[1].strip() for ln in f if ln.startswith("model name")),
                         None)
    except OSError:
        pass
    return cores, model


class CpuSample:
    """The fp64 oracle's O(mn(m+n)) row sweep (oracle.round_row_sweep, as it stands) on the
    leading r rows of the layer at full width: every row of the real layer costs about as much
    (a T_i sum over the rows above, T_i L_I, and the left-to-right pass over n columns), so
    r*n / t extrapolates to the whole layer's rounding rate. The factors come from LAPACK
    Cholesky outside the timing; numpy may use every host thread."""

    def __init__(self, wl, arrays=None):
        import numpy as np

        from two_sided_adaptive_bakron_b200.workloads import make_workload
        if arrays is None:
            arrays = make_workload(wl, device=_gram_device(wl))
        Ws, HO, HI, s, bits = arrays
        self.wl, self.bits = wl, bits
        self.Ws, self.s = Ws, s
        self.LO = _lapack_udu(HO)
        self.LI = _lapack_udu(HI)
        self.cores, self.model = cpu_info()
        self.r = 1
        del np

    def step(self, r=None):
        import oracle
        r = self.r if r is None else r
        t0 = time.perf_counter()
        oracle.round_row_sweep(self.Ws[:r], self.LO[:r, :r], self.LI, self.s[:r], self.bits)
        return time.perf_counter() - t0

    def size(self, seconds: float):
        """Grows r until one step takes at least ``seconds``; returns that step's time."""
        r = 1
        while True:
            dt = self.step(r)
            if dt >= seconds or r >= self.wl.m:
                self.r = r
                return dt
            r = min(self.wl.m, max(r + 1, int(r * min(4.0, 1.25 * seconds / max(dt, 1e-3)))))

    def describe(self, dt: float) -> dict:
        wl = self.wl
        return {"value": self.r * wl.n / dt, "unit": UNIT, "cores": self.cores,
                "kind": "oracle", "cpu_model": self.model,
                "sample": (f"oracle.round_row_sweep (fp64 numpy, up to {self.cores} threads) on "
                           f"the leading {self.r} rows x all {wl.n} columns of {wl.name}, "
                           f"{dt:.2f} s; factors from LAPACK Cholesky outside the timing; "
                           "rounding only; weights/s = rows*n/t, extrapolated to the whole "
                           "layer (per-row cost ~ n^2/2 + i n)")}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    from two_sided_adaptive_bakron_b200.workloads import WORKLOADS
    wl = WORKLOADS[args.workload]
    cs = CpuSample(wl)
    # sizing run (also the first warm-up), then the remaining warm-ups, then K timed steps
    cs.size(args.ref_seconds / 4)
    for _ in range(max(0, args.warmup - 1)):
        cs.step()
    times = [cs.step() for _ in range(args.steps)]
    t = sum(times) / len(times)
    cpu = cs.describe(t)
    v = cpu["value"]
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": wl.name, "m": wl.m, "n": wl.n, "bits": wl.bits,
                       "sample_rows": cs.r, "sample_cols": wl.n},
            "cpu_baseline": cpu,
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run(args):
    import torch
    import numpy as np

    ws, rank, local = _dist()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())

    from two_sided_adaptive_bakron_b200 import bakron as bk
    from two_sided_adaptive_bakron_b200.workloads import (WORKLOADS, make_layer_samples,
                                                          make_workload)
    wl = WORKLOADS[args.workload]
    m, n = wl.m, wl.n
    samples = None   # --hessian: (X, G) on the device, their host copies, the Gram shapes
    if args.hessian:
        Ws_np, X_np, G_np, s_np, bits = make_layer_samples(wl)
        if X_np is None or G_np is None:
            raise SystemExit(f"--hessian needs both sample matrices; {wl.name} has an "
                             "identity factor")
        samples = ((torch.from_numpy(X_np).to(dev), torch.from_numpy(G_np).to(dev)),
                   (X_np, G_np),
                   {"gram_I": (n, X_np.shape[0]), "gram_O": (m, G_np.shape[0])})
        HO = torch.empty((m, m), dtype=torch.float32, device=dev)
        HI = torch.empty((n, n), dtype=torch.float32, device=dev)
        HO_np = HI_np = None
        ws_g = bk.workspace(max(bk.bakron_damped_gram_workspace_bytes(X_np.shape[0], n),
                                bk.bakron_damped_gram_workspace_bytes(G_np.shape[0], m)), dev)
        del X_np, G_np
    else:
        Ws_np, HO_np, HI_np, s_np, bits = make_workload(wl, device=str(dev))
        HO = torch.from_numpy(HO_np).to(dev)
        HI = torch.from_numpy(HI_np).to(dev)
    Ws = torch.from_numpy(Ws_np).to(dev)
    sc = torch.from_numpy(s_np).to(dev)
    solver = bk.Solver(m, n, dev)
    stream = torch.cuda.current_stream(dev)

    # ---- per-call timing events on the launching stream (device-timed breakdown)
    names = (["gram_I", "gram_O"] if args.hessian else []) + \
        (["rotate", "unrotate"] if args.incoherence else []) + ["ldl_O", "ldl_I", "round", "loss"]

    seed = 0x5EED if args.rounding == "stochastic" else None
    quant = {}
    s_in = s_np          # the grid steps the step reads (per row, or per row and group)
    if args.group_size or args.codebook:
        if seed is not None or args.incoherence:
            raise SystemExit("stochastic Q and incoherence processing take the per-row grid")
        gs = min(args.group_size or n, n)
        book = normal_codebook(bits) if args.codebook == "normal" else None
        top = 1.0 if book is not None else (1 << (bits - 1)) - 0.5
        G = (n + gs - 1) // gs
        sg = np.stack([np.abs(Ws_np[:, g * gs:(g + 1) * gs]).max(axis=1) for g in range(G)],
                      axis=1) / np.float32(top)
        s_in = np.ascontiguousarray(sg, dtype=np.float32)
        sc = torch.from_numpy(s_in).to(dev)
        quant = {"group_size": gs, "codebook": book}
    if args.incoherence:
        quant = {"incoherence": (0x1C0, 0x1C1)}

    def factors(X, G, timing):
        # H_I from the tokens, H_O from the gradient rows, into the buffers the solve reads
        for nm, A, H in (("gram_I", X, HI), ("gram_O", G, HO)):
            ev = timing.get(nm) if timing else None
            if ev is not None:
                ev[0].record(stream)
            rc = bk.bakron_damped_gram(A, wl.damp, H, ws_g, solver.status, stream)
            if rc != 0:
                raise bk.BakronError(rc, "bakron_damped_gram")
            if ev is not None:
                ev[1].record(stream)

    def step(evs=None):
        timing = None if evs is None else dict(zip(names, evs))
        if samples is not None:
            factors(samples[0][0], samples[0][1], timing)
        solver.run(Ws, HO, HI, sc, bits, stream, timing=timing, seed=seed, **quant)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = bk.bakron_read_status(solver.status, stream)
    if st != 0:
        raise bk.BakronError(st, "warm-up")

    evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
            for _ in names] for _ in range(args.steps)]
    l0 = bk.bakron_kernel_launches()
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        t_start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        t_end.record(stream)
        torch.cuda.synchronize()
    launches = bk.bakron_kernel_launches() - l0
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), dev)
    st = bk.bakron_read_status(solver.status, stream)
    if st != 0:
        raise bk.BakronError(st, "timed region")
    ms_step = ms_total / args.steps
    value = whole_job_value(ws, m, n, ms_step)
    per = {nm: statistics.mean(evs[k][i][0].elapsed_time(evs[k][i][1]) for k in range(args.steps))
           for i, nm in enumerate(names)}

    e2e = None
    if not args.no_e2e:
        e2e = _e2e(args, torch, bk, solver, stream, dev, ws, m, n, bits, Ws, HO, HI, sc,
                   Ws_np, HO_np, HI_np, s_in, seed,
                   (samples[1], samples[0], factors) if samples is not None else None, quant)
    return _report(args, torch, bk, wl, ws, rank, m, n, bits, per, ms_step, value, launches,
                   clk, e2e, None if samples is not None else (Ws_np, HO_np, HI_np, s_np, bits),
                   samples[2] if samples is not None else None)


def _e2e(args, torch, bk, solver, stream, dev, ws, m, n, bits, Ws, HO, HI, sc,
         Ws_np, HO_np, HI_np, s_np, seed, hess=None, quant=None):
    """Same metric through the public API with host buffers: every step copies its inputs
    from pinned host memory to the device (W*, the scales and either H_O, H_I or, with
    --hessian, the samples X and G), runs the whole path, and copies the codes and the loss
    back. A step's input copies run on a copy stream into one of two device input sets while
    the previous step computes, and its results are copied device to device into a staging
    buffer and read back on a third stream while the next step computes (the copy engines and
    the SMs work at the same time); every copy of every step lies inside the timed region."""
    hW = torch.from_numpy(Ws_np).pin_memory()
    hs = torch.from_numpy(s_np).pin_memory()
    if hess is None:
        h_in = (torch.from_numpy(HO_np).pin_memory(), torch.from_numpy(HI_np).pin_memory())
        shapes = (HO, HI)
    else:
        (X_np, G_np), (Xd, Gd), factors = hess
        h_in = (torch.from_numpy(X_np).pin_memory(), torch.from_numpy(G_np).pin_memory())
        shapes = (Xd, Gd)
    # two device input sets: (W*, scales, the two factor inputs)
    sets = [(torch.empty_like(Ws), torch.empty_like(sc), torch.empty_like(shapes[0]),
             torch.empty_like(shapes[1])) for _ in range(2)]
    hcodes = torch.empty((m, n), dtype=torch.int8).pin_memory()
    hloss = torch.empty((1,), dtype=torch.float64).pin_memory()
    dcodes = torch.empty((m, n), dtype=torch.int8, device=dev)     # staging for the read-back
    dloss = torch.empty((1,), dtype=torch.float64, device=dev)
    h2d = sum(x.numel() * x.element_size() for x in (hW, hs) + h_in)
    d2h = m * n + 8
    copy_stream = torch.cuda.Stream(device=dev)
    back_stream = torch.cuda.Stream(device=dev)
    staged, read_back = torch.cuda.Event(), torch.cuda.Event()
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    consumed = [torch.cuda.Event(), torch.cuda.Event()]
    used = [False, False]

    def prefetch(b):
        # set b may be overwritten once the step that read it has finished
        if used[b]:
            copy_stream.wait_event(consumed[b])
        with torch.cuda.stream(copy_stream):
            for d_, h_ in zip(sets[b], (hW, hs) + h_in):
                d_.copy_(h_, non_blocking=True)
        copied[b].record(copy_stream)

    def run_steps(k_steps):
        prefetch(0)
        for k in range(k_steps):
            b = k & 1
            stream.wait_event(copied[b])
            if k + 1 < k_steps:
                prefetch(b ^ 1)
            dW2, ds2, d0, d1 = sets[b]
            if hess is None:
                solver.run(dW2, d0, d1, ds2, bits, stream, seed=seed, **(quant or {}))
            else:
                factors(d0, d1, None)
                solver.run(dW2, HO, HI, ds2, bits, stream, seed=seed, **(quant or {}))
            consumed[b].record(stream)
            used[b] = True
            # the staging buffer is free once the previous step's read-back has finished
            if k > 0:
                stream.wait_event(read_back)
            dcodes.copy_(solver.codes, non_blocking=True)
            dloss.copy_(solver.loss, non_blocking=True)
            staged.record(stream)
            back_stream.wait_event(staged)
            with torch.cuda.stream(back_stream):
                hcodes.copy_(dcodes, non_blocking=True)
                hloss.copy_(dloss, non_blocking=True)
            read_back.record(back_stream)

    run_steps(1)
    torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_stream.wait_event(e0)        # the first prefetch starts inside the timed region
    run_steps(args.steps)
    stream.wait_event(read_back)      # the last read-back ends inside the timed region
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    e2e_value = whole_job_value(ws, m, n, e2e_ms)
    return {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h}


# DRAM bytes (read + written) of one round_kernel launch per workload, from one ncu capture of
# the current kernel version (dram__bytes_read.sum + dram__bytes_write.sum; 1 pass on the
# 4096 x 14336 bench command, part of --set full on 4096^2); reported as the roofline's
# traffic. Emptied whenever the kernel changes, until it is captured again.
ROUND_TRAFFIC_BYTES: dict = {(4096, 14336): 33.565061e9 + 3.765866e9,
                             (4096, 4096): 3.261406e9 + 0.878998e9}


def _roofline(per, m, n, rounding="nearest", gram_dims=None, ms_step=None):
    """Roofline of the step's dominant kernel, round_kernel (one launch per step that runs the
    whole rounding solve: the largest single kernel and the largest share of the launch
    list), on its algorithmic work. The factorisation of H_I takes about as long, but as
    hundreds of short launches (diagonal blocks, panel and trailing-update GEMMs).

    The contractions run as 3xTF32 on the tensor cores (three tf32 MMAs per fp32-accurate
    product), so their peak is the measured dense bf16 rate x the nominal tf32/bf16 ratio
    (1.125 / 2.25 PFLOP/s) / 3, using the sustained bf16 figure since every call is timed
    inside a step that runs for tens of milliseconds.
    """
    peaks, kind = _peaks()
    bf16 = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops", 1400.0)))
    peak = bf16 * 0.5 / 3.0
    work = {
        "ldl_O": m ** 3 / 3.0, "ldl_I": n ** 3 / 3.0,        # U D U^T: d^3/3 flops
        "round": float(m) * n * (m + n),                       # triangular pushes, 2 flop/MAC
        "loss": 2.0 * min(m, n) ** 2 * max(m, n) + float(m) * n * max(m, n),
    }
    for k, (d, K) in (gram_dims or {}).items():       # a Gram: d (d + 1) / 2 K multiply-adds
        work[k] = float(d) * (d + 1) * K
    t = per["round"] * 1e-3
    achieved = work["round"] / t / 1e12
    return {"bound": "tensor", "kernel": "round_kernel", "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": ROUND_TRAFFIC_BYTES.get((m, n)) if rounding == "nearest" else None,
            "peak_source": (f"{kind} sustained bf16 {bf16:.1f} TFLOP/s x 0.5 (tf32/bf16 "
                            "nominal) / 3 (3xTF32), fp32-equivalent flops"),
            "work_flops": work["round"],
            # the solver benchmark's own count, the dense-equivalent 2 m n (m + n), over the
            # round kernel's time alone and over the whole step (both factorisations, the
            # round and the loss)
            "round_nominal_frac": 2.0 * work["round"] / t / 1e12 / peak,
            "step_nominal_frac": (2.0 * work["round"] / (ms_step * 1e-3) / 1e12 / peak
                                  if ms_step else None),
            "others_tflops": {k: work[k] / (per[k] * 1e-3) / 1e12 for k in per
                              if k in work and k != "round"},
            # the transforms are HBM-bound: 4 passes (read + write) per matrix, plus the grid
            # steps' read of W~
            "others_gbs": {k: b / (per[k] * 1e-3) / 1e9 for k, b in
                           (("rotate", 32.0 * (m * n + m * m + n * n) + 4.0 * m * n),
                            ("unrotate", 32.0 * m * n)) if k in per}}


def _report(args, torch, bk, wl, ws, rank, m, n, bits, per, ms_step, value, launches, clk,
            e2e, arrays, gram_dims=None):
    roofline = _roofline(per, m, n, args.rounding, gram_dims, ms_step)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cs = CpuSample(wl, arrays)
        cs.size(args.ref_seconds / 4)
        cpu = cs.describe(cs.step())
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": wl.name, "m": m, "n": n, "bits": bits,
                           "rounding": args.rounding, "hessian": bool(args.hessian),
                           "group_size": args.group_size or None,
                           "codebook": args.codebook, "incoherence": bool(args.incoherence),
                           "parallelism": f"replicas x{ws}" if ws > 1 else "single",
                           "l2": "inputs larger than L2 (H_I alone is "
                                 f"{4 * n * n / 2**20:.0f} MiB), no flush"},
                "breakdown_ms": per,
                "round_weights_per_s": m * n / (per["round"] * 1e-3),
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": int(launches), "clocks": clk.summary()}
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=12.0)
    ap.add_argument("--rounding", default="nearest", choices=["nearest", "stochastic"])
    ap.add_argument("--hessian", action="store_true")
    ap.add_argument("--group-size", type=int, default=0)
    ap.add_argument("--codebook", default=None, choices=["normal"])
    ap.add_argument("--incoherence", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run(args)


if __name__ == "__main__":
    sys.exit(main())
