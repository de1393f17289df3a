"""The multi-rank bench logic on CPU with two gloo ranks: every rank reports its own
device time, the job is timed by the slowest rank, and the whole-job rate counts the
units of all ranks (one independent session per rank, no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    local_ms = [400.0, 700.0][rank]
    ms_max = bench.max_over_ranks(local_ms)
    rate = bench.whole_job_rate(10, 4, world, ms_max)
    dist.barrier()
    q.put((rank, ms_max, rate))
    dist.destroy_process_group()


def test_two_gloo_ranks_time_by_the_slowest_and_sum_the_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_max, rate in got:
        assert ms_max == 700.0                      # the slower rank decides
        assert rate == pytest.approx(4 * 10 * 2 / 0.7)


def test_single_process_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(12.5) == 12.5
    assert bench.whole_job_rate(10, 4, 1, 1000.0) == pytest.approx(40.0)
