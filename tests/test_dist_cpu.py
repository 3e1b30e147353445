"""World-size-2 checks of the per-rank host logic, on CPU with gloo: the
slowest rank's time is reported by every rank, barriers pair up, the KV-head
shards cover the heads exactly once, and the overlap matrix pooled over the
ranks' index sets (integer counts, one all-reduce) equals the single-process
matrix bit for bit."""

import os
import socket

import numpy as np
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
        # rank 0's policy reaches every rank (sequence shards run the same layers)
        pol = D.broadcast_policy((1, 0, 0, 1, 0) if rank == 0 else None)
        assert pol == (1, 0, 0, 1, 0)
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


def _profiled_sets(L=7, B=3, Hkv=4, k=6, nb=20, seed=5):
    """Synthetic profiled index sets [L, B, Hkv, k] with some -1 padding."""
    rng = np.random.default_rng(seed)
    t = np.full((L, B, Hkv, k), -1, dtype=np.int32)
    for l in range(L):
        for b in range(B):
            for h in range(Hkv):
                m = k - (b == 2) * 2
                t[l, b, h, :m] = rng.choice(nb, size=m, replace=False)
    return t


def _pool_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from kv_cache_sparsity_b200 import hylra as H
        H.load()
        sets = _profiled_sets()
        L, B, Hkv, k = sets.shape
        heads = D.shard(Hkv, rank, world)
        mine = sets[:, :, heads.start:heads.stop].reshape(L, -1, k)
        M = D.pooled_similarity(H, mine)
        q.put((rank, list(heads), M.tobytes()))
    finally:
        torch.distributed.destroy_process_group()


def test_two_ranks_pool_the_overlap_matrix_exactly():
    from kv_cache_sparsity_b200 import build as hbuild
    from kv_cache_sparsity_b200 import hylra as H
    from oracle import hylra_oracle as O
    hbuild.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_pool_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    sets = _profiled_sets()
    L, B, Hkv, k = sets.shape
    assert sorted(res[0][1] + res[1][1]) == list(range(Hkv))
    whole = O.similarity_matrix(sets.reshape(L, -1, k))
    assert res[0][2] == res[1][2] == whole.tobytes()


def test_single_process_fallbacks():
    assert not D.dist_on()
    assert D.broadcast_policy([1, 0, 1]) == (1, 0, 1)
    assert D.max_over_ranks(2.0) == 2.0
    assert list(D.shard(5, 0, 1)) == list(range(5))
    assert [len(D.shard(10, r, 4)) for r in range(4)] == [2, 3, 2, 3]


@pytest.mark.parametrize("packed", [False, True])
def test_head_shards_hold_the_whole_layers_values(packed):
    """A rank's KV-head shard of a layer (and of a later step's query) is the
    same slice of values as in the whole layer, so sharded ranks compute
    exactly what one GPU computes for those heads."""
    from kv_cache_sparsity_b200 import workloads as W
    w = W.custom("shard", batch=2, layers=2, seqlens=(300, 129), num_q_heads=8,
                 num_kv_heads=4, topk=2, packed=packed, seed=9)
    q, K, V = W.layer_inputs(w, 1)
    for world in (2, 4):
        for rank in range(world):
            heads = D.shard(w.num_kv_heads, rank, world)
            qs, Ks, Vs = W.layer_inputs(w, 1, heads=heads)
            sl = slice(heads.start * w.group, heads.stop * w.group)
            assert torch.equal(qs, q[:, sl])
            if packed:
                assert torch.equal(Ks, K[heads.start:heads.stop])
                assert torch.equal(Vs, V[heads.start:heads.stop])
            else:
                assert torch.equal(Ks, K[:, heads.start:heads.stop])
                assert torch.equal(Vs, V[:, heads.start:heads.stop])
            assert torch.equal(W.step_query(w, 1, 2, heads=heads), W.step_query(w, 1, 2)[:, sl])
