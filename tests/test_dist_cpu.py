"""The multi-replica bookkeeping of bench.py on two gloo ranks on the CPU: the slowest rank's
time is the job's, throughput counts every rank's tokens, and every rank agrees."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        local_total_ms = [12.0, 15.0][rank]  # rank 1 is the slow one
        worst = bench.max_over_ranks(local_total_ms)
        ms, value = bench.job_throughput(worst, steps=10, world=world, tokens_per_rank=16)
        dist.barrier()
        out.put((rank, worst, ms, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, worst, ms, value in res:
        assert worst == 15.0
        assert ms == pytest.approx(1.5)
        assert value == pytest.approx(2 * 16 / 1.5e-3)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.job_throughput(20.0, 10, 1, 16) == pytest.approx((2.0, 8000.0))
