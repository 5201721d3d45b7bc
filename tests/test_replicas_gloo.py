"""The multi-GPU path shards sequences over ranks and only reduces the timing.
These run two gloo ranks on the CPU: sharding covers every sequence exactly
once, the max/sum reductions see every rank, and a rank that raises does not
leave the others hanging (a short process-group timeout ends their collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from long_context_decode_swa_b200 import replicas


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    replicas.init("gloo", timeout_s=30)
    try:
        w, r, _ = replicas.env_rank()
        mine = list(replicas.shard(13, w, r))
        slowest = replicas.max_over_ranks(1.5 + r)
        units = replicas.sum_over_ranks(len(mine))
        replicas.barrier()
        q.put((r, mine, slowest, units))
    finally:
        replicas.shutdown()


def _failing_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank))
    replicas.init("gloo", timeout_s=5)
    try:
        if rank == 1:
            raise RuntimeError("rank 1 fails before its collective")
        try:
            replicas.max_over_ranks(1.0)
            q.put((rank, "returned"))
        except Exception as e:  # the peer never joins: the collective ends with an error
            q.put((rank, type(e).__name__))
    finally:
        replicas.shutdown()


def test_shard_covers_every_sequence_once():
    for total in (0, 1, 7, 512):
        for world in (1, 2, 3, 8):
            seen = [i for r in range(world) for i in replicas.shard(total, world, r)]
            assert seen == list(range(total))
            sizes = [len(replicas.shard(total, world, r)) for r in range(world)]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        replicas.shard(4, 2, 2)


def test_two_gloo_ranks_reduce_timing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, m0, u0), (r1, s1, m1, u1) = results
    assert s0 + s1 == list(range(13))
    assert m0 == m1 == 2.5
    assert u0 == u1 == 13


def test_failed_rank_does_not_hang_the_other():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    rank, outcome = q.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
    assert rank == 0 and outcome != "returned"
    assert procs[1].exitcode != 0
