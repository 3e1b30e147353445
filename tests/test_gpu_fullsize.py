"""GPU parity at the full sizes of the five named workloads, in the launch
configuration the benchmark uses (same library calls, one CTA per SM).

* Layers 0 and 1 of each bf16 workload: sampled sequences recomputed by the
  oracle (all their heads).
* The policy path of the three DP workloads: the GPU's profiling step (every
  layer a reset layer, all layers resident as in the benchmark) -> overlap
  matrix -> DP policy, against the oracle's OWN profiling of every layer,
  sequence and KV head -> its overlap matrix -> its DP policy, bit for bit.
* The hybrid step of every bf16 workload under its policy, walked by
  oracle.decode_step on sampled sequences (every layer's output, and the
  indices of every reset layer).

Every index set's gap certificate is recorded and printed at the end of the
session with the number of near-tie swaps."""

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


SAMPLES = {  # sequences checked against the oracle
    "llama8b_32k": [0],
    "llama8b_b8_64k": [0, 5],
    "llama8b_128k": [0],
    "ragged16": None,  # shortest, longest and one in between
}


def _samples(w):
    s = SAMPLES[w.name]
    if s is not None:
        return s
    order = sorted(range(w.batch), key=lambda b: w.seqlens[b])
    return [order[0], order[len(order) // 2], order[-1]]


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["llama8b_32k", "llama8b_b8_64k", "llama8b_128k", "ragged16"])
def test_full_and_reuse_layers_at_full_size(name):
    w = W.config(name)
    run = T.Runner(w)
    q0, K0, V0 = W.layer_inputs(w, 0, "cuda")
    out0, tk0 = run.full(q0, K0, V0)
    assert run.status() == 0
    out0, tkn = out0.cpu().numpy(), tk0.cpu().numpy()
    for b in _samples(w):
        o_ref, S32, tk_ref = T.oracle_full(w, q0, K0, V0, b)
        T.check_out(out0[b], o_ref, "bf16", f"{name} full b={b}")
        for h in range(w.num_kv_heads):
            T.check_topk_certified(name, tkn[b, h], tk_ref[h], S32[h], w.topk,
                                   f"{name} b={b} h={h}")
    del K0, V0
    _free()
    q1, K1, V1 = W.layer_inputs(w, 1, "cuda")
    out1 = run.reuse(q1, K1, V1, tk0).cpu().numpy()
    assert run.status() == 0
    for b in _samples(w):
        ref = T.oracle_reuse(w, q1, K1, V1, b, tkn[b])
        T.check_out(out1[b], ref, "bf16", f"{name} reuse b={b}")
    del K1, V1
    _free()


def _walk(w, run, layers, policy, config):
    """The hybrid step under `policy` on the GPU, against oracle.decode_step
    on the sampled sequences."""
    L, B, Hkv, k = w.layers, w.batch, w.num_kv_heads, w.topk
    qs, Ks, Vs = [l[0] for l in layers], [l[1] for l in layers], [l[2] for l in layers]
    topk = torch.full((L, B, Hkv, k), -7, dtype=torch.int32, device="cuda")
    outs = [run.new_out() for _ in range(L)]
    H.decode_step(run.shape, policy, qs, Ks, Vs, run.seqlens, outs, topk, run.ws)
    assert run.status() == 0
    tk = topk.cpu().numpy()
    got = [o.cpu().numpy() for o in outs]
    del outs
    for l in range(L):
        if not policy[l]:
            assert np.all(tk[l] == -7), f"reuse layer {l} wrote its index slot"
    for b in _samples(w):
        o_ref, tk_ref = O.decode_step(policy, T.SequenceLayers(w, layers, b), [w.seqlens[b]], k)
        for l in range(L):
            T.check_out(got[l][b], o_ref[l][0], "bf16", f"{config} hybrid layer {l} b={b}")
            if policy[l]:
                # exact unless the oracle's scores hold a near tie (certified)
                S32, _ = O.layer_topk(qs[l][b].double().cpu().numpy(), T.seq_arrays(w, Ks[l], b),
                                      w.seqlens[b], k)
                for h in range(Hkv):
                    T.check_topk_certified(config, tk[l, b, h], tk_ref[l][0, h], S32[h], k,
                                           f"{config} hybrid layer {l} b={b} h={h}")


@pytest.mark.parametrize("name", ["llama8b_32k", "llama8b_b8_64k", "ragged16"])
def test_dp_policy_from_profiling_matches_oracle_and_hybrid_step(name):
    """HyLRA summary §2.2: profiling run (every layer full) -> overlap matrix
    -> DP policy.  The GPU's policy must equal the one the oracle derives from
    its own profiling, bit for bit; then the hybrid step under it is walked
    against the oracle."""
    w = W.config(name)
    L, B, Hkv, k = w.layers, w.batch, w.num_kv_heads, w.topk
    run = T.Runner(w)
    layers = [W.layer_inputs(w, l, "cuda") for l in range(L)]
    qs, Ks, Vs = [l[0] for l in layers], [l[1] for l in layers], [l[2] for l in layers]
    topk = torch.full((L, B, Hkv, k), -7, dtype=torch.int32, device="cuda")
    outs = [run.new_out() for _ in range(L)]
    H.decode_step(run.shape, (1,) * L, qs, Ks, Vs, run.seqlens, outs, topk, run.ws)
    assert run.status() == 0
    del outs
    gpu_sets = topk.cpu().numpy().reshape(L, B * Hkv, k)
    del topk

    # the oracle's own profiling: every layer, sequence and KV head
    orc_sets = np.full((L, B * Hkv, k), -1, dtype=np.int32)
    swaps = 0
    for l in range(L):
        qn = qs[l].double().cpu().numpy()
        for b in range(B):
            S32, tk = O.layer_topk(qn[b], T.seq_arrays(w, Ks[l], b), w.seqlens[b], k)
            orc_sets[l, b * Hkv:(b + 1) * Hkv] = tk
            for h in range(Hkv):
                swaps += T.check_topk_certified(name + " profiling", gpu_sets[l, b * Hkv + h],
                                                tk[h], S32[h], k, f"{name} l={l} b={b} h={h}")
    M_orc = O.similarity_matrix(orc_sets)
    M_gpu = H.similarity(gpu_sets)
    if swaps == 0:
        assert M_gpu.tobytes() == M_orc.tobytes()
    assert M_gpu.tobytes() == O.similarity_matrix(gpu_sets).tobytes()
    policy, R, S = H.dp_policy(M_gpu, w.theta)
    assert (policy, R, S) == O.dp_policy(M_gpu, w.theta)
    assert tuple(policy) == tuple(O.dp_policy(M_orc, w.theta)[0]), "policy differs from the oracle's"
    assert 1 < R < L, f"degenerate policy {policy}"
    print(f"{name}: policy {''.join('R' if x else 'U' for x in policy)} ({R} resets), "
          f"{swaps} near-tie swaps in profiling")
    _walk(w, run, layers, tuple(policy), name + " hybrid step")
    del layers, qs, Ks, Vs
    _free()


def test_128k_fixed_policy_hybrid_step_matches_oracle():
    """The 128K workload's fixed policy (a reset every fourth layer)."""
    w = W.config("llama8b_128k")
    run = T.Runner(w)
    layers = [W.layer_inputs(w, l, "cuda") for l in range(w.layers)]
    _walk(w, run, layers, w.policy, "llama8b_128k hybrid step")
    del layers
    _free()
