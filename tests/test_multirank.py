"""The multi-rank host logic of the benchmark on CPU: two gloo ranks (world size 2).

The solver runs as independent replicas (one layer per GPU, no collective on the data path);
the only cross-rank steps are the timing reduction (the slowest rank's time, on every rank)
and the barriers around the timed region. The reference arm runs on rank 0 only.
"""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench._dist()
        ms_local = 10.0 + 5.0 * rank            # rank 1 is the slow one
        ms = bench.max_over_ranks(ms_local, "cpu")
        dist.barrier()
        value = bench.whole_job_value(ws, 4096, 14336, ms)
        out[rank] = (ws, r, local, ms, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert sorted(out.keys()) == [0, 1]
    for rank in range(world):
        ws, r, local, ms, value = out[rank]
        assert (ws, r, local) == (2, rank, rank)
        assert ms == 15.0                          # both ranks see the max
        assert value == pytest.approx(2 * 4096 * 14336 / 15e-3)


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.whole_job_value(1, 10, 20, 2.0) == pytest.approx(100000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        workload = "down_4096x14336"
        steps = 1
        warmup = 3
        ref_seconds = 1.0
    assert bench.run_reference(Args()) == 0      # returns at once: no work, no output
