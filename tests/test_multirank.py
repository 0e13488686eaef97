"""Host logic of bench.py's multi-GPU form (one process per GPU, independent replicas) on CPU:
two gloo ranks must agree on the max of their step times and on the whole-job throughput."""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        total_ms = 100.0 + 25.0 * rank                      # rank 1 is the slower replica
        slowest = bench.max_over_ranks(total_ms, dist)
        value = bench.job_throughput(world, 16384, 10, slowest)
        dist.barrier()
        out.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_rank_and_the_whole_job():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [125.0, 125.0]
    # 2 replicas x 16,384 tokens x 10 steps in the slowest rank's 125 ms
    assert res[0][2] == pytest.approx(2 * 16384 * 10 / 0.125)
    assert res[0][2] == res[1][2]


def test_single_process_is_the_identity():
    import bench

    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.job_throughput(1, 16, 4, 2.0) == pytest.approx(32000.0)
