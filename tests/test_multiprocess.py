"""The N > 1 bench path on CPU with two gloo ranks: replicas report their own device time and
the job rate uses the slowest rank (max over ranks), with no data exchanged."""
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


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, _ = bench.dist_env()
        assert (r, w) == (rank, world)
        ms, rate = bench.whole_job_rate(10.0 * (rank + 1), 120, world, "cpu")
        q.put((rank, ms, rate))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_whole_job_rate_uses_slowest_rank(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = 10.0 * world
    for _, ms, rate in res:
        assert ms == slowest
        assert abs(rate - world * 120 / (slowest / 1e3)) < 1e-6


def test_single_rank_needs_no_process_group():
    import bench
    ms, rate = bench.whole_job_rate(4.0, 10, 1)
    assert ms == 4.0 and abs(rate - 2500.0) < 1e-9
