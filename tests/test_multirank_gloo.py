"""The benchmark's multi-rank logic on CPU with gloo, world size 2.

Each rank codes its own matrix (independent problems: no collective on the
data path); the only collective is the max over ranks of the timed seconds,
and the reported value is (units per rank * world) / slowest time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    secs = [1.5, 2.5][rank]
    m = bench.max_over_ranks(secs)
    rate = bench.aggregate_throughput(1000.0, m, world)
    r, w, l = bench.dist_env()
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, m, rate, r, w, l))


def test_max_over_ranks_and_aggregate_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, rate, r, w, l in res:
        assert m == 2.5
        assert rate == pytest.approx(2000.0 / 2.5)
        assert (r, w, l) == (rank, 2, rank)


def test_single_rank_helpers_without_process_group():
    import bench
    assert bench.max_over_ranks(3.0) == 3.0
    assert bench.aggregate_throughput(10.0, 2.0, 1) == 5.0
