"""Shared helpers for the GPU parity tests: run the CUDA path through the
C-ABI binding and the fp64 oracle on the same seeded inputs, and compare."""

from __future__ import annotations

import math

import numpy as np
import torch

from kv_cache_sparsity_b200 import hylra as H
from kv_cache_sparsity_b200 import workloads as W
from oracle import hylra_oracle as O

# Output tolerance for bf16 K/V against the fp64 oracle (attention outputs).
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
# fp32 inputs: fp32 accumulation and a hardware exp2 (a few ulp).
F32_MAX_ABS = 1e-4
F32_MEAN_ABS = 1e-5
# Two ranks may swap only if their oracle fp32 scores are this close.
NEAR_TIE_REL = 1e-5


class DeviceLayer:
    """One layer's inputs on the GPU plus the shape struct and buffers."""

    def __init__(self, w: W.Workload, q, K, V, device="cuda"):
        self.w = w
        self.q = q.to(device).contiguous()
        self.K = K.to(device).contiguous()
        self.V = V.to(device).contiguous()


def shape_for(w: W.Workload, seq_offsets_dev=None, kv_capacity=None) -> H.Shape:
    dtype = H.BF16 if w.dtype == "bf16" else H.FP32
    if w.packed:
        return H.make_shape(w.batch, w.num_q_heads, w.num_kv_heads, w.topk, w.max_seqlen,
                            dtype=dtype, kv_capacity=0, total_tokens=w.total_tokens,
                            seq_offsets=seq_offsets_dev)
    cap = w.max_seqlen if kv_capacity is None else kv_capacity
    return H.make_shape(w.batch, w.num_q_heads, w.num_kv_heads, w.topk, w.max_seqlen,
                        dtype=dtype, kv_capacity=cap)


class Runner:
    """Buffers for one workload shape on the GPU."""

    def __init__(self, w: W.Workload, kv_capacity=None, device="cuda"):
        self.w = w
        self.dev = device
        self.seqlens = torch.tensor(w.seqlens, dtype=torch.int32, device=device)
        self.offs = None
        if w.packed:
            self.offs = torch.tensor(W.seq_offsets(w)[:-1], dtype=torch.int64, device=device)
        self.shape = shape_for(w, self.offs, kv_capacity)
        nbytes = H.workspace_bytes(self.shape)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        H.workspace_init(self.ws)

    def new_out(self):
        w = self.w
        return torch.full((w.batch, w.num_q_heads, w.head_dim), float("nan"),
                          dtype=torch.float32, device=self.dev)

    def new_topk(self):
        w = self.w
        return torch.full((w.batch, w.num_kv_heads, w.topk), -7, dtype=torch.int32,
                          device=self.dev)

    def full(self, q, K, V):
        out, tk = self.new_out(), self.new_topk()
        H.decode_full(self.shape, q, K, V, self.seqlens, out, tk, self.ws)
        return out, tk

    def reuse(self, q, K, V, topk_in):
        out = self.new_out()
        H.decode_reuse(self.shape, q, K, V, self.seqlens, topk_in, out, self.ws)
        return out

    def status(self) -> int:
        torch.cuda.synchronize()
        return H.read_status(self.ws, clear=True)


def seq_arrays(w: W.Workload, t: torch.Tensor, b: int) -> np.ndarray:
    """[Hkv, n_b, d] fp64 numpy copy of sequence b of K or V."""
    return W.per_sequence(w, t, b).double().cpu().numpy()


def oracle_full(w, q, K, V, b):
    """Oracle reset layer for sequence b: (out [Hq,d], S32 [Hkv,NB], topk [Hkv,k])."""
    n = w.seqlens[b]
    return O.full_layer(q[b].double().cpu().numpy(), seq_arrays(w, K, b), seq_arrays(w, V, b), n,
                        w.topk)


def oracle_reuse(w, q, K, V, b, topk_b):
    n = w.seqlens[b]
    return O.reuse_attention(q[b].double().cpu().numpy(), seq_arrays(w, K, b),
                             seq_arrays(w, V, b), n, topk_b)


def check_out(got: np.ndarray, ref: np.ndarray, dtype: str, what=""):
    err = np.abs(got.astype(np.float64) - ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx, mean = float(err.max()), float(err.mean())
    if dtype == "bf16":
        assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, f"{what}: max {mx:.3g} mean {mean:.3g}"
    else:
        assert mx <= F32_MAX_ABS and mean <= F32_MEAN_ABS, f"{what}: max {mx:.3g} mean {mean:.3g}"
    return mx, mean


def check_topk(got: np.ndarray, ref: np.ndarray, S32: np.ndarray, what=""):
    """Exact match, except swaps between ranks whose oracle scores are a
    near-tie (relative gap < NEAR_TIE_REL); returns the number of such swaps."""
    got = np.asarray(got)
    ref = np.asarray(ref)
    if np.array_equal(got, ref):
        return 0
    # every rank must hold a block whose oracle score equals (to a near-tie)
    # the oracle's block at that rank, and the -1 padding must agree
    assert np.array_equal(got < 0, ref < 0), f"{what}: padding differs {got} vs {ref}"
    assert len(set(got[got >= 0].tolist())) == int((got >= 0).sum()), f"{what}: duplicates {got}"
    swaps = 0
    for i, (a, b) in enumerate(zip(got, ref)):
        if a == b:
            continue
        sa, sb = float(S32[a]), float(S32[b])
        rel = abs(sa - sb) / max(abs(sb), 1e-300)
        assert rel < NEAR_TIE_REL, (f"{what}: rank {i}: got block {a} (score {sa!r}) "
                                    f"expected {b} (score {sb!r})")
        swaps += 1
    return swaps


def min_gap(S32_rows, k) -> float:
    return min((O.topk_gap(r, k) for r in S32_rows), default=math.inf)


# Gap certificates of the top-k checks, per configuration, printed at the end
# of the session (conftest.pytest_terminal_summary): for each index set the
# oracle's smallest relative gap between consecutive fp32 scores of ranks
# 1..k'+1 (oracle.topk_gap).  A set whose gap is below NEAR_TIE_REL is a
# near tie: the kernel's fp32 sums (another summation order) may swap those
# ranks, so such a set is reported as "near-tie, unpinned".  A gap of exactly
# 0 is a tie the tests build on purpose (identical blocks): the kernel then
# computes identical scores and the tie rule (lower block first) decides.
CERTIFICATES: dict = {}


def check_topk_certified(config: str, got, ref, S32_h, k: int, what=""):
    """check_topk plus the set's gap certificate, recorded under `config`.
    A swap is accepted only inside a near tie; returns the swap count."""
    swaps = check_topk(got, ref, S32_h, what)
    gap = O.topk_gap(S32_h, k)
    assert swaps == 0 or gap < NEAR_TIE_REL, f"{what}: swap with certificate {gap}"
    c = CERTIFICATES.setdefault(config, {"sets": 0, "min_gap": math.inf, "near_ties": 0,
                                         "exact_ties": 0, "swaps": 0})
    c["sets"] += 1
    c["min_gap"] = min(c["min_gap"], gap)
    c["near_ties"] += int(0.0 < gap < NEAR_TIE_REL)
    c["exact_ties"] += int(gap == 0.0)
    c["swaps"] += swaps
    return swaps


def certificate_lines():
    out = []
    for name in sorted(CERTIFICATES):
        c = CERTIFICATES[name]
        state = "near-tie, unpinned" if c["near_ties"] else "pinned"
        ties = (f", {c['exact_ties']} sets with exactly equal scores (tie rule)"
                if c["exact_ties"] else "")
        out.append(f"{name}: {c['sets']} index sets, min relative gap {c['min_gap']:.3g}, "
                   f"{c['near_ties']} near-tie sets{ties}, {c['swaps']} swaps ({state})")
    return out


class SequenceLayers:
    """The layers of one sequence b as the fp64 arrays oracle.decode_step
    takes (q [1, Hq, d], K and V [1, Hkv, n_b, d]), converted when a layer is
    read, so that only one layer is held in host memory at a time."""

    def __init__(self, w: W.Workload, layers, b: int):
        self.w, self.layers, self.b = w, layers, b

    def __len__(self):
        return len(self.layers)

    def __getitem__(self, l):
        q, K, V = self.layers[l]
        return (q[self.b:self.b + 1].double().cpu().numpy(), seq_arrays(self.w, K, self.b)[None],
                seq_arrays(self.w, V, self.b)[None])
