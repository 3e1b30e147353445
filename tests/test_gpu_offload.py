"""Index-guided offloading (HyLRA summary §2.4): a reuse layer whose cache is
in pinned host memory gathers only its reused blocks into a device staging
cache and attends over them.  The result must equal the device-resident
reuse layer bit for bit (same values, same kernel arithmetic), and through it
the oracle; a decode step with offloaded reuse layers must equal the plain
step."""

import numpy as np
import pytest
import torch

from kv_cache_sparsity_b200 import build as hbuild
from kv_cache_sparsity_b200 import hylra as H
from kv_cache_sparsity_b200 import workloads as W

import hylra_testlib as T

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    hbuild.build()
    H.load()


def _pinned(t):
    return t.detach().cpu().pin_memory()


def _stage(run):
    n = H.stage_bytes(run.shape) // 2
    return (torch.empty(n, dtype=torch.bfloat16, device="cuda"),
            torch.empty(n, dtype=torch.bfloat16, device="cuda"))


CASES = [
    W.custom("off_dense", batch=2, layers=2, seqlens=(5000, 1700), num_q_heads=32,
             num_kv_heads=8, topk=16, seed=41),
    W.custom("off_packed", batch=3, layers=2, seqlens=(300, 4096, 1000), num_q_heads=8,
             num_kv_heads=2, topk=8, packed=True, seed=42),
    W.custom("off_group8", batch=1, layers=2, seqlens=(2500,), num_q_heads=16, num_kv_heads=2,
             topk=6, seed=43),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_staged_reuse_equals_device_reuse(w):
    run = T.Runner(w)
    q0, K0, V0 = (t.cuda() for t in W.layer_inputs(w, 0, "cpu"))
    _, tk = run.full(q0, K0, V0)
    q1, K1, V1 = W.layer_inputs(w, 1, "cpu")
    q1 = q1.cuda()
    ref = run.reuse(q1, K1.cuda(), V1.cuda(), tk)
    assert run.status() == 0
    Kh, Vh = _pinned(K1), _pinned(V1)
    Ks, Vs = _stage(run)
    Ks.fill_(float("nan"))
    Vs.fill_(float("nan"))
    H.gather_blocks(run.shape, Kh, Vh, run.seqlens, tk, Ks, Vs)
    out = run.new_out()
    H.decode_reuse_staged(run.shape, q1, Ks, Vs, run.seqlens, tk, out, run.ws)
    assert run.status() == 0
    assert torch.equal(out, ref)
    # and through it the oracle
    tkn = tk.cpu().numpy()
    for b in range(w.batch):
        o_ref = T.oracle_reuse(w, q1, K1, V1, b, tkn[b])
        T.check_out(out[b].cpu().numpy(), o_ref, "bf16", f"{w.name} staged b={b}")


def test_staged_reuse_skips_unused_and_invalid_slots():
    w = W.custom("off_ragged", batch=2, layers=2, seqlens=(129, 2000), num_q_heads=8,
                 num_kv_heads=2, topk=8, seed=44)
    run = T.Runner(w)
    q, K, V = (t.cuda() for t in W.layer_inputs(w, 1, "cpu"))
    tk = torch.tensor([[[1, 0, -1, -1, -1, -1, -1, -1], [0, -1, 1, -1, -1, -1, -1, -1]],
                       [[15, 3, 7, -1, 2, -1, -1, -1], [0, 1, 2, 3, 4, 5, 6, 15]]],
                      dtype=torch.int32, device="cuda")
    ref = run.reuse(q, K, V, tk)
    Ks, Vs = _stage(run)
    H.gather_blocks(run.shape, _pinned(K), _pinned(V), run.seqlens, tk, Ks, Vs)
    out = run.new_out()
    H.decode_reuse_staged(run.shape, q, Ks, Vs, run.seqlens, tk, out, run.ws)
    assert run.status() == 0
    assert torch.equal(out, ref)


def _stage2(run):
    """Two staging slots each for K and V (the offloaded step's prefetch)."""
    n = H.stage_bytes(run.shape)  # bytes of one slot = elements of two bf16 slots
    return (torch.empty(n, dtype=torch.bfloat16, device="cuda"),
            torch.empty(n, dtype=torch.bfloat16, device="cuda"))


@pytest.mark.parametrize("policy,offloaded", [
    ((1, 0, 0, 1, 0, 0, 0), (0, 1, 1, 0, 1, 1, 1)),
    # slots reused several times, a device-resident reuse layer between
    # offloaded ones, two reset layers in a row
    ((1, 0, 0, 0, 1, 1, 0, 0, 0, 0), (0, 1, 0, 1, 0, 0, 1, 1, 1, 1)),
])
def test_offloaded_step_equals_device_step(policy, offloaded):
    """The prefetching offloaded step equals the device-resident step bit for
    bit, eagerly and replayed from a CUDA graph.  Layer 0 makes each
    sequence's newest block rank first, so the offloaded layers copy it again
    after their preceding layer."""
    L = len(policy)
    w = W.custom("off_step", batch=2, layers=L, seqlens=(6000, 2600 - 31), num_q_heads=32,
                 num_kv_heads=8, topk=16, seed=45)
    run = T.Runner(w)
    layers = [list(W.layer_inputs(w, l, "cpu")) for l in range(w.layers)]
    u = W.structure(w).u
    for b, n in enumerate(w.seqlens):
        last = (n - 1) // 128 * 128
        K0 = layers[0][1]
        K0[b, :, last:n] = (K0[b, :, last:n].float() + 9.0 * u[b][:, None, :]).to(K0.dtype)
    qs = [l[0].cuda() for l in layers]
    Kd = [l[1].cuda() for l in layers]
    Vd = [l[2].cuda() for l in layers]
    outs_d = [run.new_out() for _ in range(w.layers)]
    topk_d = torch.full((w.layers, w.batch, w.num_kv_heads, w.topk), -7, dtype=torch.int32,
                        device="cuda")
    H.decode_step(run.shape, policy, qs, Kd, Vd, run.seqlens, outs_d, topk_d, run.ws)
    assert run.status() == 0
    Ko = [Kd[l] if not offloaded[l] else _pinned(layers[l][1]) for l in range(w.layers)]
    Vo = [Vd[l] if not offloaded[l] else _pinned(layers[l][2]) for l in range(w.layers)]
    outs_o = [run.new_out() for _ in range(w.layers)]
    topk_o = torch.full_like(topk_d, -7)
    Ks, Vs = _stage2(run)
    H.decode_step_offload(run.shape, policy, qs, Ko, Vo, offloaded, run.seqlens, outs_o,
                          topk_o, Ks, Vs, run.ws)
    assert run.status() == 0
    assert torch.equal(topk_o, topk_d)
    assert np.all(topk_d[0, :, :, 0].cpu().numpy() == np.array([[(n - 1) // 128] * 8
                                                                for n in w.seqlens]))
    for l in range(w.layers):
        assert torch.equal(outs_o[l], outs_d[l]), f"layer {l}"
    # replayed from a CUDA graph (the copy stream's work becomes graph nodes)
    for o in outs_o:
        o.fill_(float("nan"))
    topk_o.fill_(-7)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        H.decode_step_offload(run.shape, policy, qs, Ko, Vo, offloaded, run.seqlens, outs_o,
                              topk_o, Ks, Vs, run.ws, stream=torch.cuda.current_stream())
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert run.status() == 0
    assert torch.equal(topk_o, topk_d)
    for l in range(w.layers):
        assert torch.equal(outs_o[l], outs_d[l]), f"graph layer {l}"


def test_offloaded_reset_layer_is_rejected():
    w = W.custom("off_bad", batch=1, layers=2, seqlens=(1024,), num_q_heads=8, num_kv_heads=2,
                 topk=4, seed=46)
    run = T.Runner(w)
    layers = [_ for _ in (W.layer_inputs(w, l, "cuda") for l in range(2))]
    Ks, Vs = _stage2(run)
    outs = [run.new_out() for _ in range(2)]
    topk = torch.full((2, 1, 2, 4), -1, dtype=torch.int32, device="cuda")
    with pytest.raises(H.HylraError) as e:
        H.decode_step_offload(run.shape, (1, 0), [l[0] for l in layers], [l[1] for l in layers],
                              [l[2] for l in layers], (1, 0), run.seqlens, outs, topk, Ks, Vs,
                              run.ws)
    assert e.value.code == -1


def test_reuse_beyond_the_cluster_grid_limit():
    """B * Hkv = 65,536 (one more than a grid's y extent): reuse layers take
    the streaming kernel + merge kernel path, plain and staged."""
    w = W.custom("wide", batch=1024, layers=2, seqlens=(256,) * 1024, num_q_heads=64,
                 num_kv_heads=64, topk=2, seed=47)
    run = T.Runner(w)
    q0, K0, V0 = W.layer_inputs(w, 0, "cuda")
    _, tk = run.full(q0, K0, V0)
    assert run.status() == 0
    del K0, V0
    q1, K1, V1 = W.layer_inputs(w, 1, "cuda")
    out = run.reuse(q1, K1, V1, tk)
    assert run.status() == 0
    tkn = tk.cpu().numpy()
    for b in (0, 517, 1023):
        o_ref = T.oracle_reuse(w, q1, K1, V1, b, tkn[b])
        T.check_out(out[b].cpu().numpy(), o_ref, "bf16", f"wide reuse b={b}")
    Kh, Vh = _pinned(K1), _pinned(V1)
    del K1, V1
    torch.cuda.empty_cache()
    Ks, Vs = _stage(run)
    H.gather_blocks(run.shape, Kh, Vh, run.seqlens, tk, Ks, Vs)
    out_s = run.new_out()
    H.decode_reuse_staged(run.shape, q1, Ks, Vs, run.seqlens, tk, out_s, run.ws)
    assert run.status() == 0
    assert torch.equal(out_s, out)
