"""The multi-rank host logic of bench.py on CPU: two gloo ranks.

Requests are independent, so `bench.py --gpus N` runs one replica per GPU and
only reduces timing across ranks: the slowest rank's elapsed time (all-reduce
MAX) and the whole-job rate (all ranks' steps over that time).
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [12.5, 20.0, 7.0, 15.0][rank]
        mx = bench.slowest_rank_ms(local, world)
        q.put((rank, mx, bench.job_value(world, 100, mx)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_slowest_rank_and_job_rate(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = max([12.5, 20.0, 7.0, 15.0][:world])
    for rank, mx, value in out:
        assert mx == want
        assert value == pytest.approx(world * 100 / (want / 1000.0))


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.slowest_rank_ms(3.0, 1) == 3.0
    assert bench.job_value(1, 10, 5.0) == pytest.approx(2000.0)
