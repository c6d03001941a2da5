"""The benchmark's multi-process path on the CPU: two ranks over gloo (127.0.0.1).

bench.py runs one process per GPU under torchrun; every rank streams the same work
(independent problems, no collective on the data path), the step time is the maximum over
ranks and the reported value is the whole job's bytes over that time (weak scaling).  These
tests run that host logic with world_size 2 without a GPU: the max-over-ranks reduction,
the barrier, the job rate, and that the reference arm does its work on rank 0 only.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [2.0, 3.5][rank]                      # rank 1 is the slow one
        bench.barrier(world)
        ms = bench.max_over_ranks(local_ms, world)
        gbs = bench.job_gbs(1e9, ms, world)
        # the reference arm returns at once on every rank but 0 (no oracle work, no output)
        args = type("A", (), {"steps": 1, "warmup": 0})()
        if rank != 0:
            bench.run_reference(args, rank, world)
        bench.barrier(world)
        out.put((rank, ms, gbs))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_job_rate():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=5) for _ in range(2))
    for rank, ms, gbs in res:
        assert ms == pytest.approx(3.5)                   # both ranks see the slowest rank's time
        assert gbs == pytest.approx(2 * 1e9 / 3.5e-3 / 1e9)  # the job's bytes over that time


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.25, 1) == 1.25
    assert bench.job_gbs(2e9, 1.0, 1) == pytest.approx(2000.0)
