"""GPU parity: the CUDA path (through the C-ABI) against the fp64 oracle on
the same seeded inputs, at sizes that span several work units and a ragged
tail, plus the edge cases of the method."""

import dataclasses

import numpy as np
import pytest
import torch

from kv_cache_sparsity_b200 import build as hbuild
from kv_cache_sparsity_b200 import hylra as H
from kv_cache_sparsity_b200 import workloads as W
from oracle import hylra_oracle as O

import hylra_testlib as T

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    hbuild.build()
    H.load()


def _layer(w, layer=0):
    q, K, V = W.layer_inputs(w, layer, device="cpu")
    return q.cuda(), K.cuda(), V.cuda()


def _full_and_check(w, layer=0, kv_capacity=None, inputs=None):
    run = T.Runner(w, kv_capacity=kv_capacity)
    q, K, V = inputs if inputs is not None else _layer(w, layer)
    out, tk = run.full(q, K, V)
    assert run.status() == 0
    out, tk = out.cpu().numpy(), tk.cpu().numpy()
    swaps = 0
    for b in range(w.batch):
        o_ref, S32, tk_ref = T.oracle_full(w, q, K, V, b)
        T.check_out(out[b], o_ref, w.dtype, f"{w.name} b={b}")
        for h in range(w.num_kv_heads):
            swaps += T.check_topk_certified(w.name, tk[b, h], tk_ref[h], S32[h], w.topk,
                                            f"{w.name} b={b} h={h}")
    return run, (q, K, V), out, tk, swaps


CASES = [
    W.custom("b1_h8_2_n4096", seqlens=(4096,), num_q_heads=8, num_kv_heads=2, topk=8),
    W.custom("b3_dense_ragged", batch=3, seqlens=(1000, 128, 1), num_q_heads=8, num_kv_heads=2,
             topk=4, seed=3),
    W.custom("packed_ragged", batch=4, seqlens=(300, 2048, 129, 5000), num_q_heads=32,
             num_kv_heads=8, topk=16, packed=True, seed=4),
    W.custom("group1", seqlens=(2000,), num_q_heads=4, num_kv_heads=4, topk=6, seed=5),
    W.custom("group2", seqlens=(3000,), num_q_heads=8, num_kv_heads=4, topk=6, seed=6),
    W.custom("group8", seqlens=(2500,), num_q_heads=16, num_kv_heads=2, topk=6, seed=7),
    W.custom("group5", batch=2, seqlens=(2200, 700), num_q_heads=10, num_kv_heads=2, topk=6,
             seed=32),
    W.custom("group7", seqlens=(1900,), num_q_heads=14, num_kv_heads=2, topk=5, seed=33),
    W.custom("iid_bf16", seqlens=(6000,), num_q_heads=8, num_kv_heads=2, topk=8,
             structure="iid", seed=8),
    W.custom("many_heads", batch=2, seqlens=(9000, 7000), num_q_heads=64, num_kv_heads=16,
             topk=12, seed=9),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_full_layer_matches_oracle(w):
    _full_and_check(w)


def test_tiny_fp32_config_step_matches_oracle():
    """The small fp32 configuration: 4 layers, fixed policy [R, U, U, R]."""
    w = W.config("tiny")
    run = T.Runner(w)
    layers = [_layer(w, l) for l in range(w.layers)]
    topk = torch.full((w.layers, w.batch, w.num_kv_heads, w.topk), -7, dtype=torch.int32,
                      device="cuda")
    outs = [run.new_out() for _ in range(w.layers)]
    H.decode_step(run.shape, w.policy, [l[0] for l in layers], [l[1] for l in layers],
                  [l[2] for l in layers], run.seqlens, outs, topk, run.ws)
    assert run.status() == 0
    np_layers = [(q.double().cpu().numpy(), K.double().cpu().numpy(), V.double().cpu().numpy())
                 for q, K, V in layers]
    o_ref, tk_ref = O.decode_step(w.policy, np_layers, w.seqlens, w.topk)
    tk = topk.cpu().numpy()
    for l in range(w.layers):
        T.check_out(outs[l].cpu().numpy()[0], o_ref[l][0], "fp32", f"tiny layer {l}")
        if w.policy[l]:
            _, S32, _ = T.oracle_full(w, *layers[l], 0)
            for h in range(w.num_kv_heads):
                assert T.check_topk_certified("tiny", tk[l, 0, h], tk_ref[l][0, h], S32[h], w.topk,
                                              f"tiny l={l}") == 0


def test_fp32_ragged_packed():
    w = W.custom("fp32_packed", batch=3, seqlens=(777, 130, 2049), num_q_heads=6, num_kv_heads=2,
                 topk=5, dtype="fp32", packed=True, structure="iid", seed=11)
    _full_and_check(w)


def test_dense_tail_rows_may_hold_nan():
    """Rows past n_b in a dense cache are not part of the sequence: even NaN
    there must not reach the output."""
    w = W.custom("nan_tail", batch=2, seqlens=(1000, 300), num_q_heads=8, num_kv_heads=2, topk=4,
                 seed=12)
    q, K, V = _layer(w)
    K = K.clone()
    V = V.clone()
    for b, n in enumerate(w.seqlens):
        K[b, :, n:] = float("nan")
        V[b, :, n:] = float("nan")
    _full_and_check(w, inputs=(q, K, V))
    run = T.Runner(w)
    idx = torch.tensor([[[7, 0, 3, -1], [7, 1, -1, -1]], [[2, 0, 1, -1], [0, 2, -1, -1]]],
                       dtype=torch.int32, device="cuda")
    out = run.reuse(q, K, V, idx).cpu().numpy()
    assert run.status() == 0
    for b in range(2):
        ref = T.oracle_reuse(w, q, K, V, b, idx[b].cpu().numpy())
        T.check_out(out[b], ref, "bf16", f"nan_tail reuse b={b}")


def test_capacity_larger_than_longest_sequence():
    w = W.custom("cap", batch=2, seqlens=(640, 1500), num_q_heads=8, num_kv_heads=2, topk=4,
                 seed=13)
    q, K, V = _layer(w)
    cap = 2048
    K2 = torch.zeros(2, 2, cap, 128, dtype=K.dtype, device="cuda")
    V2 = torch.zeros_like(K2)
    K2[:, :, :K.shape[2]] = K
    V2[:, :, :V.shape[2]] = V
    _full_and_check(w, kv_capacity=cap, inputs=(q, K2, V2))


@pytest.mark.parametrize("w", CASES[:3] + [CASES[6], CASES[7]] +
                         [W.custom("fp32r", seqlens=(1500, 4000), batch=2,
                                   dtype="fp32", structure="iid", seed=14)],
                         ids=lambda w: w.name)
def test_reuse_layer_matches_oracle(w):
    """Reuse with the indices the full kernel produced for another layer."""
    w = dataclasses.replace(w, layers=2)
    run = T.Runner(w)
    q0, K0, V0 = _layer(w, 0)
    q1, K1, V1 = _layer(w, 1)
    _, tk = run.full(q0, K0, V0)
    out = run.reuse(q1, K1, V1, tk).cpu().numpy()
    assert run.status() == 0
    tkn = tk.cpu().numpy()
    for b in range(w.batch):
        ref = T.oracle_reuse(w, q1, K1, V1, b, tkn[b])
        T.check_out(out[b], ref, w.dtype, f"{w.name} reuse b={b}")


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_reuse_with_every_block_equals_full(dtype):
    w = W.custom("allblocks", batch=2, seqlens=(1300, 700), num_q_heads=8, num_kv_heads=2,
                 topk=11, dtype=dtype, seed=15)
    run = T.Runner(w)
    q, K, V = _layer(w)
    out_f, _ = run.full(q, K, V)
    nb = [(n + 127) // 128 for n in w.seqlens]
    idx = torch.full((2, 2, 11), -1, dtype=torch.int32)
    for b in range(2):
        for h in range(2):
            idx[b, h, :nb[b]] = torch.randperm(nb[b])
    out_r = run.reuse(q, K, V, idx.cuda())
    assert run.status() == 0
    tol = 2e-3 if dtype == "bf16" else 1e-5
    assert torch.allclose(out_r, out_f, atol=tol, rtol=0)


def test_reuse_many_blocks_per_cta():
    """k = 64 of 128 blocks over 8 KV heads: each cluster CTA takes several
    blocks with refills (the plan that also puts the warp states into a
    stage at the end to fit a third stage)."""
    w = W.custom("reuse_k64", batch=1, layers=2, seqlens=(128 * 128 - 5,), num_q_heads=32,
                 num_kv_heads=8, topk=64, seed=31)
    run = T.Runner(w)
    q0, K0, V0 = _layer(w, 0)
    q1, K1, V1 = _layer(w, 1)
    _, tk = run.full(q0, K0, V0)
    out = run.reuse(q1, K1, V1, tk).cpu().numpy()
    assert run.status() == 0
    ref = T.oracle_reuse(w, q1, K1, V1, 0, tk.cpu().numpy()[0])
    T.check_out(out[0], ref, "bf16", "reuse_k64")


def test_step_reuse_refills_the_stage_of_an_early_newest_block():
    """Inside a step a reuse layer rereads the newest cache row after its
    wait and writes it into the staged block.  Here the newest block ranks
    first (so it sits in the first stage of the first CTA) and every CTA has
    more blocks than stages, so that stage is refilled by TMA after the row
    was rewritten: the refill must land after the rewrite."""
    n = 128 * 100 - 37  # partial newest block
    w = W.custom("newest_first", batch=1, layers=2, seqlens=(n,), num_q_heads=8,
                 num_kv_heads=2, topk=64, seed=41)
    q0, K0, V0 = W.layer_inputs(w, 0, device="cpu")
    u = W.structure(w).u  # [B, Hkv, d] salient directions the queries follow
    last = (n - 1) // 128 * 128
    K0[0, :, last:n] = (K0[0, :, last:n].float() + 9.0 * u[0][:, None, :]).to(K0.dtype)
    layers = [(q0.cuda(), K0.cuda(), V0.cuda()), _layer(w, 1)]
    run = T.Runner(w)
    policy = (1, 0)
    topk = torch.full((2, 1, 2, 64), -7, dtype=torch.int32, device="cuda")
    outs = [run.new_out() for _ in range(2)]
    for _ in range(3):
        H.decode_step(run.shape, policy, [l[0] for l in layers], [l[1] for l in layers],
                      [l[2] for l in layers], run.seqlens, outs, topk, run.ws)
        assert run.status() == 0
        tk = topk.cpu().numpy()
        assert np.all(tk[0, 0, :, 0] == (n - 1) // 128), "newest block not ranked first"
        np_layers = [tuple(t.double().cpu().numpy() for t in l) for l in layers]
        o_ref, tk_ref = O.decode_step(policy, np_layers, w.seqlens, w.topk)
        assert np.array_equal(tk[0], tk_ref[0])
        for l in range(2):
            T.check_out(outs[l].cpu().numpy(), o_ref[l], "bf16", f"newest-first layer {l}")


def test_reuse_skips_minus_one_and_flags_bad_indices():
    w = W.custom("badidx", batch=1, seqlens=(1000,), num_q_heads=8, num_kv_heads=2, topk=4,
                 seed=16)
    run = T.Runner(w)
    q, K, V = _layer(w)
    idx = torch.tensor([[[3, -1, 99, 5], [-5, 2, -1, -1]]], dtype=torch.int32, device="cuda")
    out = run.reuse(q, K, V, idx).cpu().numpy()
    st = run.status()
    assert st & H.STATUS_BAD_INDEX
    ref = T.oracle_reuse(w, q, K, V, 0, np.array([[3, -1, -1, 5], [-1, 2, -1, -1]]))
    T.check_out(out[0], ref, "bf16", "badidx")


def test_reuse_flags_duplicate_indices():
    w = W.custom("dupidx", batch=1, seqlens=(1000,), num_q_heads=8, num_kv_heads=2, topk=4,
                 seed=24)
    run = T.Runner(w)
    q, K, V = _layer(w)
    idx = torch.tensor([[[3, 1, 3, -1], [0, 1, 2, 4]]], dtype=torch.int32, device="cuda")
    run.reuse(q, K, V, idx)
    assert run.status() & H.STATUS_DUP_INDEX
    idx = torch.tensor([[[3, 1, 2, -1], [0, 1, 2, 4]]], dtype=torch.int32, device="cuda")
    run.reuse(q, K, V, idx)
    assert run.status() == 0


def test_reuse_empty_selection_gives_zero():
    w = W.custom("empty_sel", batch=1, seqlens=(500,), num_q_heads=8, num_kv_heads=2, topk=3,
                 seed=17)
    run = T.Runner(w)
    q, K, V = _layer(w)
    idx = torch.full((1, 2, 3), -1, dtype=torch.int32, device="cuda")
    out = run.reuse(q, K, V, idx)
    assert run.status() == 0
    assert torch.all(out == 0)


def test_empty_sequence_and_k_beyond_blocks():
    w = W.custom("edge", batch=3, seqlens=(0, 200, 1), num_q_heads=8, num_kv_heads=2, topk=4,
                 seed=18)
    run, (q, K, V), out, tk, _ = _full_and_check(w)
    assert np.all(out[0] == 0) and np.all(tk[0] == -1)
    assert np.all(tk[1, :, 2:] == -1) and np.all(tk[2, :, 1:] == -1) and np.all(tk[2, :, 0] == 0)


def test_equal_scores_pick_lowest_indices():
    """All keys zero: every logit equal, every full block the same mass, the
    partial last block less; ranks follow block index (lower first)."""
    w = W.custom("ties", batch=1, seqlens=(128 * 9 + 50,), num_q_heads=8, num_kv_heads=2, topk=6,
                 seed=19)
    q, K, V = _layer(w)
    K = torch.zeros_like(K)
    _, _, _, tk, _ = _full_and_check(w, inputs=(q, K, V))
    assert np.all(tk[0] == np.arange(6))


def test_many_equal_scores_rank_by_block_index():
    """1000 blocks of equal mass (the merge tree); ranks must follow block
    index."""
    w = W.custom("ties_many", batch=1, seqlens=(128 * 1000,), num_q_heads=8, num_kv_heads=2,
                 topk=20, seed=25)
    q, K, V = _layer(w)
    K = torch.zeros_like(K)
    _, _, _, tk, _ = _full_and_check(w, inputs=(q, K, V))
    assert np.all(tk[0] == np.arange(20))


@pytest.mark.parametrize("nblocks", [200, 256, 257])
def test_equal_scores_rank_by_block_index(nblocks):
    """Every block of equal mass, on both sides of the one-key-per-thread
    selection limit (256 blocks): ranks must follow block index."""
    w = W.custom(f"ties_{nblocks}", batch=1, seqlens=(128 * nblocks,), num_q_heads=8,
                 num_kv_heads=2, topk=24, seed=27)
    q, K, V = _layer(w)
    K = torch.zeros_like(K)
    _, _, _, tk, _ = _full_and_check(w, inputs=(q, K, V))
    assert np.all(tk[0] == np.arange(24))


@pytest.mark.parametrize("nblocks,topk,dtype,structure", [
    (300, 20, "bf16", "salient"),
    (512, 32, "bf16", "iid"),
    (1000, 24, "bf16", "salient"),
    (2000, 32, "bf16", "iid"),
    (200, 30, "fp32", "iid"),
    (400, 32, "fp32", "salient"),
    (300, 40, "fp32", "iid"),
    (513, 33, "bf16", "salient"),
    (1024, 64, "bf16", "iid"),
])
def test_selection_paths_match_oracle(nblocks, topk, dtype, structure):
    """More blocks than selection threads: the merge tree of per-warp sorted
    lists for k' <= 32 (bf16: 256 threads, fp32: 128), the radix select
    above (both kernels); each with a ragged last block."""
    w = W.custom(f"sel_{nblocks}_{topk}_{dtype}", batch=1, seqlens=(128 * nblocks - 37,),
                 num_q_heads=8, num_kv_heads=2, topk=topk, dtype=dtype, structure=structure,
                 seed=60 + nblocks % 17)
    _full_and_check(w)


@pytest.mark.parametrize("nblocks,topk", [(300, 20), (700, 32), (2048, 32), (600, 48)])
def test_equal_mass_ranks_by_block_index_on_larger_paths(nblocks, topk):
    """Every full block of equal mass on the merge-tree (k' <= 32) and radix
    paths: ranks follow block index."""
    w = W.custom(f"ties_tree_{nblocks}", batch=1, seqlens=(128 * nblocks,), num_q_heads=8,
                 num_kv_heads=2, topk=topk, seed=28)
    q, K, V = _layer(w)
    K = torch.zeros_like(K)
    _, _, _, tk, _ = _full_and_check(w, inputs=(q, K, V))
    assert np.all(tk[0] == np.arange(topk))


def test_k_larger_than_the_merge_thread_count():
    """k = 300 > 256 selection threads: the radix select path."""
    w = W.custom("bigk", batch=1, seqlens=(128 * 400 - 17,), num_q_heads=8, num_kv_heads=2,
                 topk=300, structure="iid", seed=26)
    _full_and_check(w)


def test_invalid_seqlen_is_flagged_not_faulted():
    w = W.custom("badlen", batch=2, seqlens=(300, 300), num_q_heads=8, num_kv_heads=2, topk=3,
                 seed=20)
    run = T.Runner(w)
    q, K, V = _layer(w)
    run.seqlens[1] = 5000  # beyond the cache
    out, tk = run.full(q, K, V)
    st = run.status()
    assert st & H.STATUS_BAD_SEQLEN
    assert torch.all(out[1] == 0) and torch.all(tk[1] == -1)
    ref, _, tk_ref = T.oracle_full(w, q, K, V, 0)
    T.check_out(out[0].cpu().numpy(), ref, "bf16", "badlen b=0")


def test_step_hybrid_matches_oracle_walk():
    w = W.custom("step", batch=2, layers=6, seqlens=(3000, 1700), num_q_heads=8, num_kv_heads=2,
                 topk=5, seed=21)
    policy = (1, 0, 0, 1, 0, 1)
    run = T.Runner(w)
    layers = [_layer(w, l) for l in range(w.layers)]
    topk = torch.full((w.layers, 2, 2, 5), -7, dtype=torch.int32, device="cuda")
    outs = [run.new_out() for _ in range(w.layers)]
    H.decode_step(run.shape, policy, [l[0] for l in layers], [l[1] for l in layers],
                  [l[2] for l in layers], run.seqlens, outs, topk, run.ws)
    assert run.status() == 0
    np_layers = []
    for q, K, V in layers:
        np_layers.append((q.double().cpu().numpy(), K.double().cpu().numpy(),
                          V.double().cpu().numpy()))
    o_ref, tk_ref = O.decode_step(policy, np_layers, w.seqlens, w.topk)
    tk = topk.cpu().numpy()
    for l in range(w.layers):
        T.check_out(outs[l].cpu().numpy(), o_ref[l], "bf16", f"step layer {l}")
        if policy[l]:
            assert np.array_equal(tk[l], tk_ref[l]), f"layer {l}"
        else:
            assert np.all(tk[l] == -7)   # reuse layers leave their slot untouched


def test_step_in_cuda_graph_matches_eager():
    w = W.custom("graph", batch=1, layers=4, seqlens=(4096,), num_q_heads=8, num_kv_heads=2,
                 topk=8, seed=22)
    policy = (1, 0, 1, 0)
    run = T.Runner(w)
    layers = [_layer(w, l) for l in range(w.layers)]
    topk = torch.full((4, 1, 2, 8), -1, dtype=torch.int32, device="cuda")
    outs = [run.new_out() for _ in range(4)]
    args = ([l[0] for l in layers], [l[1] for l in layers], [l[2] for l in layers])
    H.decode_step(run.shape, policy, *args, run.seqlens, outs, topk, run.ws)
    torch.cuda.synchronize()
    eager = [o.clone() for o in outs]
    eager_tk = topk.clone()
    for o in outs:
        o.fill_(float("nan"))
    topk.fill_(-1)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        H.decode_step(run.shape, policy, *args, run.seqlens, outs, topk, run.ws,
                      stream=torch.cuda.current_stream())
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for a, b in zip(outs, eager):
        assert torch.equal(a, b)
    assert torch.equal(topk, eager_tk)
    assert run.status() == 0


@pytest.mark.parametrize("policy", [(1, 0, 0, 0, 1, 0, 0, 1), (1, 1, 0, 1, 0, 0, 0, 0)])
def test_graph_step_ordering_under_repeated_replays(policy):
    """Layers overlap through programmatic launch; a reuse layer must never
    read index slots before the reset layer that owns them has written them.
    The slots are poisoned with an invalid index before every replay, so an
    early read shows up in the status word (and in the outputs)."""
    w = W.custom("order", batch=1, layers=8, seqlens=(32768,), num_q_heads=32, num_kv_heads=8,
                 topk=16, seed=27)
    run = T.Runner(w)
    layers = [_layer(w, l) for l in range(w.layers)]
    args = ([l[0] for l in layers], [l[1] for l in layers], [l[2] for l in layers])
    topk = torch.full((8, 1, 8, 16), -7, dtype=torch.int32, device="cuda")
    outs = [run.new_out() for _ in range(8)]
    H.decode_step(run.shape, policy, *args, run.seqlens, outs, topk, run.ws)
    torch.cuda.synchronize()
    assert run.status() == 0
    ref = [o.clone() for o in outs]
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        topk.fill_(-7)
        H.decode_step(run.shape, policy, *args, run.seqlens, outs, topk, run.ws,
                      stream=torch.cuda.current_stream())
    for _ in range(30):
        g.replay()
    torch.cuda.synchronize()
    assert run.status() == 0
    for a, b in zip(outs, ref):
        assert torch.equal(a, b)


def test_step_host_buffers_match_device_step():
    w = W.custom("hoststep", batch=2, layers=3, seqlens=(2000, 900), num_q_heads=8,
                 num_kv_heads=2, topk=4, seed=23)
    policy = (1, 0, 1)
    run = T.Runner(w)
    layers = [_layer(w, l) for l in range(w.layers)]
    q_host = torch.stack([l[0].cpu() for l in layers]).pin_memory()
    q_dev = torch.empty_like(q_host, device="cuda")
    out_dev = torch.empty(3, 2, 8, 128, dtype=torch.float32, device="cuda")
    out_host = torch.empty(3, 2, 8, 128, dtype=torch.float32).pin_memory()
    tk_dev = torch.full((3, 2, 2, 4), -1, dtype=torch.int32, device="cuda")
    tk_host = torch.empty(3, 2, 2, 4, dtype=torch.int32).pin_memory()
    H.decode_step_host(run.shape, policy, q_host, q_dev, [l[1] for l in layers],
                       [l[2] for l in layers], run.seqlens, out_dev, out_host, tk_dev, tk_host,
                       run.ws)
    torch.cuda.synchronize()
    outs = [run.new_out() for _ in range(3)]
    tk2 = torch.full((3, 2, 2, 4), -1, dtype=torch.int32, device="cuda")
    H.decode_step(run.shape, policy, [l[0] for l in layers], [l[1] for l in layers],
                  [l[2] for l in layers], run.seqlens, outs, tk2, run.ws)
    torch.cuda.synchronize()
    assert torch.equal(out_host, torch.stack([o.cpu() for o in outs]))
    assert torch.equal(tk_host[0], tk2[0].cpu()) and torch.equal(tk_host[2], tk2[2].cpu())
    assert run.status() == 0


def test_step_host_buffers_in_a_cuda_graph():
    """The host-buffer step (its copies run on a second stream, overlapped
    with the layers) captured in a CUDA graph and replayed with new queries:
    every replay's host outputs equal the device step on the same inputs."""
    w = W.custom("hostgraph", batch=2, layers=9, seqlens=(3000, 1200), num_q_heads=8,
                 num_kv_heads=2, topk=6, seed=29)
    policy = (1, 0, 0, 1, 0, 1, 1, 0, 0)
    run = T.Runner(w)
    layers = [_layer(w, l) for l in range(w.layers)]
    K, V = [l[1] for l in layers], [l[2] for l in layers]
    L = w.layers
    q_host = torch.stack([l[0].cpu() for l in layers]).pin_memory()
    q_dev = torch.empty_like(q_host, device="cuda")
    out_dev = torch.empty(L, 2, 8, 128, dtype=torch.float32, device="cuda")
    out_host = torch.empty(L, 2, 8, 128, dtype=torch.float32).pin_memory()
    tk_dev = torch.full((L, 2, 2, 6), -1, dtype=torch.int32, device="cuda")
    tk_host = torch.empty(L, 2, 2, 6, dtype=torch.int32).pin_memory()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        H.decode_step_host(run.shape, policy, q_host, q_dev, K, V, run.seqlens, out_dev,
                           out_host, tk_dev, tk_host, run.ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        H.decode_step_host(run.shape, policy, q_host, q_dev, K, V, run.seqlens, out_dev,
                           out_host, tk_dev, tk_host, run.ws, stream=torch.cuda.current_stream())
    gen = torch.Generator().manual_seed(5)
    for rep in range(3):
        q_host.copy_(torch.randn(q_host.shape, generator=gen).to(q_host.dtype))
        out_host.fill_(float("nan"))
        tk_host.fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        outs = [run.new_out() for _ in range(L)]
        tk2 = torch.full((L, 2, 2, 6), -1, dtype=torch.int32, device="cuda")
        H.decode_step(run.shape, policy, [q_host[l].cuda() for l in range(L)], K, V, run.seqlens,
                      outs, tk2, run.ws)
        torch.cuda.synchronize()
        assert torch.equal(out_host, torch.stack([o.cpu() for o in outs])), f"replay {rep}"
        for l in range(L):
            if policy[l]:
                assert torch.equal(tk_host[l], tk2[l].cpu()), f"replay {rep} layer {l}"
    assert run.status() == 0
    del g


def test_repeated_calls_are_deterministic():
    w = CASES[2]
    run = T.Runner(w)
    q, K, V = _layer(w)
    o1, t1 = run.full(q, K, V)
    o2, t2 = run.full(q, K, V)
    assert torch.equal(o1, o2) and torch.equal(t1, t2)
    assert run.status() == 0


def test_workspace_too_small_is_rejected():
    w = CASES[0]
    run = T.Runner(w)
    q, K, V = _layer(w)
    small = run.ws[:256]
    with pytest.raises(H.HylraError) as e:
        H.decode_full(run.shape, q, K, V, run.seqlens, run.new_out(), run.new_topk(), small)
    assert e.value.code == -4


def test_bounded_waits_give_up_and_the_workspace_recovers():
    """Failure detection without a fault: with a wait limit of one SM clock
    the kernels' waits for their TMA copies (and the reuse cluster's wait for
    its peers) give up.  Each kernel then stops issuing, waits for the copies
    it already issued, finishes, and sets HYLRA_STATUS_TIMEOUT.  With the
    default limit back, the same workspace (status cleared) gives exactly the
    results of a run that never timed out."""
    w = W.custom("timeout", batch=2, layers=4, seqlens=(20000, 9000), num_q_heads=32,
                 num_kv_heads=8, topk=16, seed=51)
    run = T.Runner(w)
    layers = [_layer(w, l) for l in range(w.layers)]
    args = ([l[0] for l in layers], [l[1] for l in layers], [l[2] for l in layers])
    policy = (1, 0, 0, 1)

    def step():
        topk = torch.full((w.layers, 2, 8, 16), -7, dtype=torch.int32, device="cuda")
        outs = [run.new_out() for _ in range(w.layers)]
        H.decode_step(run.shape, policy, *args, run.seqlens, outs, topk, run.ws)
        return outs, topk

    def single_layers():
        out, tk = run.full(*layers[0])
        return [out, run.reuse(*layers[1], tk)], tk

    good = step()
    assert run.status() == 0
    good_single = single_layers()
    assert run.status() == 0
    seen = {}
    try:
        H.set_wait_limit(1)
        for name, fn in (("step", step), ("single", single_layers)):
            for _ in range(5):  # a wait gives up unless its data was already there
                fn()
                st = run.status()  # reads and clears
                # (a layer that gave up computes on whatever its stages held, so its
                # block scores may also be flagged as non-finite)
                assert st & ~(H.STATUS_TIMEOUT | H.STATUS_NONFINITE) == 0, f"{name}: {st:#x}"
                if st & H.STATUS_TIMEOUT:
                    seen[name] = True
                    break
    finally:
        H.set_wait_limit(0)
    assert seen == {"step": True, "single": True}, seen
    for fn, ref in ((step, good), (single_layers, good_single)):
        outs, tk = fn()
        assert run.status() == 0
        for a, b in zip(outs, ref[0]):
            assert torch.equal(a, b)
        assert torch.equal(tk, ref[1])


TOKEN_CASES = [
    W.custom("tok_dense", batch=2, seqlens=(3000, 700), num_q_heads=8, num_kv_heads=2, topk=6,
             seed=61),
    W.custom("tok_packed_r1", batch=3, seqlens=(1300, 129, 2500), num_q_heads=4, num_kv_heads=4,
             topk=5, packed=True, seed=62),
    W.custom("tok_fp32", batch=1, seqlens=(1000,), num_q_heads=8, num_kv_heads=2, topk=4,
             dtype="fp32", structure="iid", seed=63),
]
# Token masses: fp32 logits of 128 products (absolute error ~1e-5 in the
# log2 domain, i.e. ~1e-5 relative in the probability), a head sum built from
# the blocks' fp32 records and a hardware exp2: 1e-4 relative is ten times that.
TOKEN_RTOL = 1e-4


@pytest.mark.parametrize("w", TOKEN_CASES, ids=lambda w: w.name)
def test_token_scores_match_oracle(w):
    """Token-level profiling: per-token attention mass against the oracle;
    the host selection on the GPU's scores against the oracle's ranking rule
    (exact), and the selected tokens valid against the oracle's own scores."""
    run = T.Runner(w)
    q, K, V = _layer(w, 0)
    out_ref, tk_ref = run.full(q, K, V)
    assert run.status() == 0
    out, tk = run.new_out(), run.new_topk()
    scores = torch.full((w.batch, w.num_kv_heads, w.max_seqlen), float("nan"), device="cuda")
    H.token_scores(run.shape, q, K, V, run.seqlens, out, tk, scores, run.ws)
    assert run.status() == 0
    assert torch.equal(out, out_ref) and torch.equal(tk, tk_ref)
    sc = scores.cpu().numpy()
    ktok = 128 * w.topk
    for b in range(w.batch):
        n = w.seqlens[b]
        S32, _ = O.layer_token_topk(q[b].double().cpu().numpy(), T.seq_arrays(w, K, b), n, ktok)
        assert np.all(sc[b, :, n:] == 0.0)
        np.testing.assert_allclose(sc[b, :, :n], S32, rtol=TOKEN_RTOL, atol=1e-12)
        got = H.token_topk(sc[b, :, :n], ktok)
        for h in range(w.num_kv_heads):
            assert np.array_equal(got[h], O.topk_blocks(sc[b, h, :n], ktok))
            # valid against the oracle: no chosen token scores clearly below a
            # token left out
            kp = min(ktok, n)
            chosen = S32[h][got[h][:kp]].astype(np.float64)
            left = np.delete(S32[h], got[h][:kp]).astype(np.float64)
            if left.size:
                assert chosen.min() >= left.max() * (1 - 2 * TOKEN_RTOL)


def test_large_reuse_layer_stream_split_parity_and_index_flags():
    """A reuse layer large enough for the stream-K split over every SM (16 x
    8 heads x 16 blocks, clusters would leave SMs idle): outputs against the
    oracle, and a duplicated, an out-of-range and a -1 entry handled as on the
    cluster path (duplicate counted twice and flagged, out-of-range skipped
    and flagged, -1 skipped)."""
    w = W.custom("reuse_streamk", batch=16, layers=2, seqlens=(2176,) * 15 + (2000,),
                 num_q_heads=32, num_kv_heads=8, topk=16, seed=71)
    run = T.Runner(w)
    q0, K0, V0 = _layer(w, 0)
    q1, K1, V1 = _layer(w, 1)
    _, tk = run.full(q0, K0, V0)
    assert run.status() == 0
    out = run.reuse(q1, K1, V1, tk)
    assert run.status() == 0
    out, tkn = out.cpu().numpy(), tk.cpu().numpy()
    for b in (0, 15):
        T.check_out(out[b], T.oracle_reuse(w, q1, K1, V1, b, tkn[b]), "bf16", f"stream-K b={b}")
    bad = tkn.copy()
    bad[3, 2, 5] = bad[3, 2, 1]          # duplicate
    bad[5, 1, 0] = 17 + 999              # out of range
    bad[7, 0, 4] = -1                    # skipped
    out2 = run.reuse(q1, K1, V1, torch.from_numpy(bad).cuda())
    st = run.status()
    assert st & H.STATUS_DUP_INDEX and st & H.STATUS_BAD_INDEX
    out2 = out2.cpu().numpy()
    ref_lists = bad.copy()
    ref_lists[5, 1, 0] = -1              # the kernel skips an out-of-range block
    for b in (3, 5, 7, 0):
        T.check_out(out2[b], T.oracle_reuse(w, q1, K1, V1, b, ref_lists[b]), "bf16",
                    f"stream-K flagged b={b}")


def test_large_reuse_layer_group8_empty_sequence_and_repeat():
    """The reuse merge of the stream-K path with r = 8 q-heads per KV head
    (two float4 columns per merge thread), a sequence without tokens (no
    units: zero output) and a repeated index (counted twice, flagged): 16
    sequences x 4 KV heads x 24 reused blocks, large enough for the split
    over every SM."""
    lens = (3840, 4000, 3300, 3968, 3100, 0, 4096, 3500, 3072, 3900, 3700, 3200, 4000, 3333, 3999,
            3600)
    w = W.custom("reuse_streamk_r8", batch=16, layers=2, seqlens=lens, num_q_heads=32,
                 num_kv_heads=4, topk=24, seed=92)
    run = T.Runner(w)
    q0, K0, V0 = _layer(w, 0)
    q1, K1, V1 = _layer(w, 1)
    _, tk = run.full(q0, K0, V0)
    assert run.status() == 0
    tkn = tk.cpu().numpy()
    assert np.all(tkn[5] == -1)
    out = run.reuse(q1, K1, V1, tk)
    assert run.status() == 0
    out = out.cpu().numpy()
    assert np.all(out[5] == 0.0)
    for b in (0, 6, 15):
        T.check_out(out[b], T.oracle_reuse(w, q1, K1, V1, b, tkn[b]), "bf16", f"r8 b={b}")
    bad = tkn.copy()
    bad[6, 3, 10] = bad[6, 3, 2]  # repeated: counted twice, flagged
    out2 = run.reuse(q1, K1, V1, torch.from_numpy(bad).cuda())
    assert run.status() & H.STATUS_DUP_INDEX
    out2 = out2.cpu().numpy()
    for b in (6, 0):
        T.check_out(out2[b], T.oracle_reuse(w, q1, K1, V1, b, bad[b]), "bf16", f"r8 repeat b={b}")


def test_maximum_topk_reset_and_reuse():
    """k = HYLRA_MAX_TOPK (1024) of 1500 blocks: the radix selection at its
    largest k, and a reuse layer over 1024 blocks per head."""
    w = W.custom("maxk", batch=1, layers=2, seqlens=(128 * 1500 - 9,), num_q_heads=8,
                 num_kv_heads=2, topk=H.MAX_TOPK, structure="iid", seed=81)
    run, (q, K, V), out, tk, swaps = _full_and_check(w)
    assert np.all(tk[0] >= 0)  # k' = 1024 <= 1500 blocks: no padding
    q1, K1, V1 = _layer(w, 1)
    out1 = run.reuse(q1, K1, V1, torch.from_numpy(tk).cuda())
    assert run.status() == 0
    ref = T.oracle_reuse(w, q1, K1, V1, 0, tk[0])
    T.check_out(out1.cpu().numpy()[0], ref, "bf16", "maxk reuse")


def test_maximum_batch():
    """B = HYLRA_MAX_BATCH (1024) sequences of mixed small lengths (0 .. 300
    tokens, packed): the per-sequence prefix sums and splits at their widest;
    sampled sequences against the oracle, empty ones zero with -1 indices."""
    rng = np.random.default_rng(82)
    lens = [int(x) for x in rng.integers(0, 301, size=H.MAX_BATCH)]
    lens[5] = 0
    w = W.custom("maxbatch", batch=H.MAX_BATCH, layers=2, seqlens=lens, num_q_heads=4,
                 num_kv_heads=2, topk=2, packed=True, seed=83)
    run = T.Runner(w)
    q, K, V = _layer(w, 0)
    out, tk = run.full(q, K, V)
    assert run.status() == 0
    out, tk = out.cpu().numpy(), tk.cpu().numpy()
    assert np.all(out[5] == 0.0) and np.all(tk[5] == -1)
    for b in (0, 1, 511, 1023):
        o_ref, S32, tk_ref = T.oracle_full(w, q, K, V, b)
        T.check_out(out[b], o_ref, "bf16", f"maxbatch b={b}")
        for h in range(w.num_kv_heads):
            T.check_topk_certified("maxbatch", tk[b, h], tk_ref[h], S32[h], w.topk,
                                   f"maxbatch b={b} h={h}")
    q1, K1, V1 = _layer(w, 1)
    out1 = run.reuse(q1, K1, V1, torch.from_numpy(tk).cuda()).cpu().numpy()
    assert run.status() == 0
    assert np.all(out1[5] == 0.0)
    for b in (0, 1023):
        T.check_out(out1[b], T.oracle_reuse(w, q1, K1, V1, b, tk[b]), "bf16", f"maxbatch reuse {b}")
