"""Host logic of the multi-process benchmark path, on CPU with gloo (world size 2).

The hot path has no data-path collective (independent layers per rank); what
crosses ranks is the barrier around the timed region, the maximum of the
per-rank device times and the sharding of units.  These run here as two gloo
processes on 127.0.0.1.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

from sparse_linear_layers_bitnet_b200 import dist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    info = dist.init(backend="gloo", timeout_s=60)
    assert info.rank == rank and info.world == world
    dist.barrier()
    # per-rank device time: the job time is the slowest rank
    t = dist.max_over_ranks(10.0 + rank)
    s = dist.sum_over_ranks(1.0)
    shards = list(dist.shard(7, rank, world))
    out[rank] = (t, s, shards)
    dist.finalize()


def test_two_rank_timing_and_sharding():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 11.0
    assert out[0][1] == out[1][1] == 2.0
    assert out[0][2] + out[1][2] == list(range(7))


def test_shard_covers_everything():
    for n in (0, 1, 5, 30, 31):
        for w in (1, 2, 3, 8):
            parts = [list(dist.shard(n, r, w)) for r in range(w)]
            flat = [x for p in parts for x in p]
            assert flat == list(range(n))
            assert max(map(len, parts)) - min(map(len, parts)) <= 1


def test_single_process_is_identity(monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    info = dist.init()
    assert info.world == 1
    assert dist.max_over_ranks(3.5) == 3.5
    dist.barrier()
