"""The multi-GPU path is N independent replicas: the only cross-rank steps are the timing
barrier and a max over ranks.  Here two gloo ranks on the CPU check that every rank receives the
slowest rank's time and that the whole-job throughput counts every rank's units."""
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


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    local = [3.0, 7.5][rank]  # rank 1 is the slow one
    dist.barrier()
    m = bench.max_over_ranks(local, torch.device("cpu"), world)
    v = bench.throughput(world, 1000, 4, m)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, m, v))


def test_two_replicas_report_the_slowest_rank_and_the_whole_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    for rank, m, v in res:
        assert m == 7.5
        assert v == pytest.approx(2 * 1000 * 4 / 7.5e-3)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(2.5, torch.device("cpu"), 1) == 2.5
    assert bench.throughput(1, 10, 2, 4.0) == pytest.approx(5000.0)
