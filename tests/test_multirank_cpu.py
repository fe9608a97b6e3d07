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


def test_lpt_assignment_of_a_70b_block():
    """Every layer goes to exactly one rank; the largest load is within the LPT bound
    (average + largest item); the assignment is a pure function of the sizes."""
    import bench
    import workloads as WL
    shapes = WL.block70b_shapes()
    costs = [m * n * (m + n) for _, m, n, _ in shapes]
    for world in (1, 2, 3, 4, 8):
        owner = bench.lpt_assign(costs, world)
        assert len(owner) == len(costs) and all(0 <= r < world for r in owner)
        loads = [sum(c for c, r in zip(costs, owner) if r == q) for q in range(world)]
        assert max(loads) <= sum(costs) / world + max(costs)
        assert owner == bench.lpt_assign(costs, world)
    # two ranks: the three large layers split 2 + 1, the rest fill the lighter rank
    owner = bench.lpt_assign(costs, 2)
    big = [i for i, c in enumerate(costs) if c == max(costs)]
    assert sorted(owner[i] for i in big) == [0, 0, 1]


def _block_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads as WL
        shapes = WL.block70b_shapes()
        owner = bench.lpt_assign([m * n * (m + n) for _, m, n, _ in shapes], world)
        mine = [i for i, r in enumerate(owner) if r == rank]
        got = [None] * world
        dist.all_gather_object(got, mine)     # test only: the bench needs no exchange
        t = bench.max_over_ranks(1.0 + rank)
        q.put((rank, got, t))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_cover_the_block_once():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_block_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    shares = res[0][1]
    assert shares == res[1][1]                                  # same assignment on both ranks
    assert sorted(i for s in shares for i in s) == list(range(7))
    assert [r[2] for r in res] == [2.0, 2.0]                    # the block's time: slowest rank
