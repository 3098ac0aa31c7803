"""The multi-GPU path of the benchmark is replicas only (every rank runs the
same single-GPU step; there is no exchange on the data path).  What the ranks
do share is the timing: the job's time is the slowest rank's, and the job's
rate counts every rank's work.  Tested with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    import bench
    secs = [0.5, 0.8, 0.65][rank]
    m = bench.max_over_ranks(secs, torch.device("cpu"))
    v = bench.job_throughput(10.0, 4, world, m)
    out.put((rank, m, v))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_time_is_the_slowest_rank_and_work_counts_every_rank(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = max([0.5, 0.8, 0.65][:world])
    for rank, m, v in res:
        assert m == slowest
        assert v == pytest.approx(world * 10.0 * 4 / slowest)


def test_single_process_is_the_identity():
    import torch
    import bench
    assert bench.max_over_ranks(0.25, torch.device("cpu")) == 0.25
    assert bench.job_throughput(3.0, 2, 1, 0.5) == 12.0
