"""The N > 1 benchmark plumbing on CPU: two gloo ranks, max-over-ranks time,
whole-job throughput and balanced sharding."""

import os
import socket

import pytest
import torch.multiprocessing as mp

from bit_weight_only_lcvq_b200.replicas import Replicas, shard, throughput


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    R = Replicas(backend="gloo", timeout_s=60)
    R.barrier()
    t_max = R.max(1.0 + rank)        # rank r "took" 1 + r seconds
    total = R.sum(10.0)
    mine = list(shard(225, world, rank))
    R.close()
    q.put((rank, t_max, total, mine))


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.0, 2.0]           # both see the slowest rank
    assert [r[2] for r in res] == [20.0, 20.0]
    shards = res[0][3] + res[1][3]
    assert shards == list(range(225))                   # disjoint and complete
    assert abs(len(res[0][3]) - len(res[1][3])) <= 1


def test_throughput_and_shard_edges():
    assert throughput(100.0, 4, 2.0) == 200.0
    assert list(shard(3, 4, 3)) == [2] and list(shard(3, 4, 0)) == []
    with pytest.raises(ZeroDivisionError):
        throughput(1.0, 1, 0.0)
