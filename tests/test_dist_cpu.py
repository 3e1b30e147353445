"""World-size-2 checks of the per-rank host logic, on CPU with gloo: the
slowest rank's time is reported by every rank, barriers pair up, and the
sequence shards of a batch cover it exactly once."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from kv_cache_sparsity_b200 import dist as D


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, w = D.rank_env()
        assert (r, lr, w) == (rank, rank, world)
        assert D.dist_on()
        got = D.max_over_ranks(1.5 + rank * 2.25)
        D.barrier()
        shard = list(D.shard(7, rank, world))
        q.put((rank, got, shard))
    finally:
        torch.distributed.destroy_process_group()


def test_two_ranks_max_and_shards():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [g for _, g, _ in res] == [3.75, 3.75]
    covered = res[0][2] + res[1][2]
    assert sorted(covered) == list(range(7))


def test_single_process_fallbacks():
    assert not D.dist_on()
    assert D.max_over_ranks(2.0) == 2.0
    assert list(D.shard(5, 0, 1)) == list(range(5))
    assert [len(D.shard(10, r, 4)) for r in range(4)] == [2, 3, 2, 3]
