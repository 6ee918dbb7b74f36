"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the job's time is the max
over ranks, the job's rate counts every rank's bytes, and only rank 0 reports."""

import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from datetime import timedelta

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench

        ms_local = [3.0, 5.0][rank]
        ms = bench.max_over_ranks(ms_local)
        rate = bench.job_gbs(world, 1e9, ms)
        # the reference arm: rank 0 alone prints its line; the others return without work
        buf = io.StringIO()
        if rank != 0:
            class A:
                gpus, steps, warmup = world, 1, 3
            with redirect_stdout(buf):
                bench.reference_arm(A())
        out.put((rank, ms, rate, buf.getvalue()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, rate, printed in got:
        assert ms == 5.0  # the slowest rank's time, on every rank
        assert rate == pytest.approx(2 * 1e9 / 5e-3 / 1e9)  # both ranks' bytes over that time
        if rank != 0:
            assert printed == ""


def test_max_over_ranks_without_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(2.5) == 2.5
    assert bench.job_gbs(1, 2e9, 1000.0) == pytest.approx(2.0)
