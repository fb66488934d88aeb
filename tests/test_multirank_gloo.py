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


def _shard_worker(rank, world, port, q):
    """Row-sharded calibration, exchange step: every rank holds the fp64 sums
    of |z| over its rows; gather_partial_sums must give every rank all of them
    in rank order (the sums here come from the oracle's rotation: no GPU)."""
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    import synth
    import vector_codebook_codec_b200 as qamw
    from oracle import codec
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    spec = synth.tiny().specs[0]
    W = synth.make_matrix(spec)
    act = synth.act_for(spec)
    bounds = [0, 100, spec.M]                     # uneven shards
    lo, hi = bounds[rank], bounds[rank + 1]
    _, _, Y = codec.rotated_rows(W[lo:hi], act, spec.alpha, spec.block, spec.seed)
    mine = np.sqrt(np.sum(codec.pairs(Y) ** 2, axis=2)).sum(axis=0)
    got = qamw.gather_partial_sums(torch.from_numpy(mine))
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got.numpy()))


def test_sharded_calibration_exchange_gloo():
    import numpy as np

    import synth
    from oracle import codec
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    spec = synth.tiny().specs[0]
    W = synth.make_matrix(spec)
    act = synth.act_for(spec)
    _, _, Y = codec.rotated_rows(W, act, spec.alpha, spec.block, spec.seed)
    whole = np.sqrt(np.sum(codec.pairs(Y) ** 2, axis=2)).sum(axis=0)
    assert res[0].shape == (2, spec.K // 2)
    assert np.array_equal(res[0], res[1])                     # every rank has the same table
    assert np.allclose(res[0][0] + res[0][1], whole, rtol=1e-12, atol=0)
