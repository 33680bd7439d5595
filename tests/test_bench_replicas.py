"""The multi-process plumbing of bench.py on CPU: two gloo ranks (replicas only -- the path
has no exchange step).  Each rank reports its own step time; the job's time is the maximum
over ranks and the job's rate counts every rank's bytes."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import sys
    from datetime import timedelta

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        ms = [2.0, 5.0][rank]  # rank 1 is the slower replica
        m = bench.max_over_ranks(ms, torch.device("cpu"), world)
        rate = bench.job_rate(1e9, m, world)
        out.put((rank, m, rate))
        # the reference leg: rank 0 alone runs it; other ranks return at once
        if rank != 0:
            class A:
                fmt, batch, gpus, steps, warmup = "q8_0", 4, world, 1, 3
            assert bench.run_reference(A, rank, world) is None
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_max_time_and_job_rate():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    res = sorted(out.get(timeout=5) for _ in range(2))
    for rank, m, rate in res:
        assert m == 5.0                       # every rank sees the slowest rank's time
        assert rate == pytest.approx(2 * 1e9 / 5e-3 / 1e9)  # both ranks' bytes / max time
