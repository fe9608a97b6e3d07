"""Multi-rank host logic of bench.py on CPU: two gloo ranks, no GPU.

Each rank rounds its own independent layer (no data-path collective); the only
collectives are the barrier and the max-over-ranks reduction of the timing."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = bench.max_over_ranks(10.0 + 5.0 * rank)          # rank 1 is the slower one
        dist.barrier()
        q.put((rank, ms, bench.rank_seed(rank), bench.aggregate_value(4096, 4096, world, ms)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert [g[1] for g in got] == [15.0, 15.0]                 # max over ranks on every rank
    assert len({g[2] for g in got}) == world                   # independent layers
    assert got[0][3] == pytest.approx(2 * 4096 * 4096 / 15e-3)  # whole-job entries/s


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
