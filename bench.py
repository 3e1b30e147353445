"""HyLRA decode-attention benchmark (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is one decode step of the whole hot path: every layer of the model,
a reset layer running full attention + block scoring + top-k, a reuse layer
attending over the blocks the most recent reset layer selected, under the
policy the DP derives from a profiling run (all layers full) of the same
synthetic workload.  Inputs are resident in HBM before timing starts; each
step streams more bytes than the 126 MB L2 holds.  The default workload is
the largest one that fits one GPU (ragged16: 16 sequences of 8K-128K tokens,
all 32 layer caches resident).

With N GPUs (torchrun) there is no collective in the step.  Default
(--shard batch, "scaling": "weak"): one global batch of N x B sequences,
rank r running its own B (the configured workload's shapes, its own seed;
rank 0's is the configured workload) under the policy rank 0 derives, which
every rank receives.  --shard heads ("scaling": "strong"): rank r holds the
KV heads shard(Hkv, r, N) of every sequence of the one workload, and the
profiled overlap matrix is pooled exactly over the ranks (integer counts, one
all-reduce), so every rank runs the policy a single GPU derives.

value        = device time per hybrid decode step (us), max over ranks
e2e          = the same step through the C-ABI host-buffer entry point
               (q copied host->device, outputs device->host, inside the timing)
roofline     = the reset layer (streaming + merge kernels): K+V bytes of one
               layer on this GPU over its average time in the all-reset step
reuse_layer  = a reuse layer's K+V bytes over its average time in a step of one
               reset layer followed by reuse layers
cpu_baseline / --impl reference = the fp64 oracle, single-threaded on the host,
               on a bounded sample (one reset and one reuse layer of one KV head
               of every sequence), scaled to a whole step
"""

from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_sparsity_b200 import build as hbuild  # noqa: E402
from kv_cache_sparsity_b200 import dist as D  # noqa: E402
from kv_cache_sparsity_b200 import workloads as W  # noqa: E402

METRIC = ("decode-attention µs/step & KV HBM GB/s vs ~8 TB/s; HyLRA vs full speedup")
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------- helpers

def workload_desc(w: W.Workload) -> str:
    lens = (f"context {w.seqlens[0]}" if len(set(w.seqlens)) == 1
            else f"ragged contexts {min(w.seqlens)}..{max(w.seqlens)} (sum {w.total_tokens})")
    pol = "DP policy theta=%g" % w.theta if w.policy is None else "fixed policy"
    return (f"{w.name}: batch {w.batch}, {w.layers} layers, {w.num_q_heads} q / "
            f"{w.num_kv_heads} KV heads, head_dim {w.head_dim}, {w.dtype} K/V, {lens}, "
            f"block 128, top-k {w.topk}, {pol}, {'packed' if w.packed else 'dense'} layout")


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def ncu_traffic(kernel_tag: str, workload: str):
    """Per-launch DRAM bytes from a committed ncu summary, if it was taken
    on the current kernel source (null otherwise)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}_{workload}.txt")
    if not os.path.exists(path):
        return None
    src = b""
    for fn in ("hylra_kernels.cuh", "hylra_device.cuh"):
        with open(os.path.join(ROOT, "kv_cache_sparsity_b200", "csrc", fn), "rb") as f:
            src += f.read()
    sha = hashlib.sha256(src).hexdigest()[:16]
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line:
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256_16") != sha:
        return None
    try:
        return float(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock/throttle samples while the GPU works."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.15)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9 or (self.uuid and parts[0] != self.uuid):
                    continue
                rows.append(parts)
        os.unlink(self.path)
        busy = [r for r in rows if _num(r[4]) and _num(r[4]) > 0] or rows
        sm = [_num(r[1]) for r in busy if _num(r[1])]
        smax = [_num(r[2]) for r in rows if _num(r[2])]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in busy for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(busy)}


def _num(x):
    try:
        return float(x)
    except ValueError:
        return None


# ----------------------------------------------------------------- our arm

class Model:
    """All layers of one synthetic workload resident on this GPU: the KV
    heads ``heads`` of every sequence (all of them on one GPU)."""

    def __init__(self, w: W.Workload, H, resident_layers: int, heads: range):
        self.w, self.H, self.heads = w, H, heads
        dev = "cuda"
        self.nkv = len(heads)
        self.nq = self.nkv * w.group
        self.seqlens = torch.tensor(w.seqlens, dtype=torch.int32, device=dev)
        self.offs = (torch.tensor(W.seq_offsets(w)[:-1], dtype=torch.int64, device=dev)
                     if w.packed else None)
        dtype = H.BF16 if w.dtype == "bf16" else H.FP32
        if w.packed:
            self.shape = H.make_shape(w.batch, self.nq, self.nkv, w.topk, w.max_seqlen,
                                      dtype=dtype, total_tokens=w.total_tokens,
                                      seq_offsets=self.offs)
        else:
            self.shape = H.make_shape(w.batch, self.nq, self.nkv, w.topk, w.max_seqlen,
                                      dtype=dtype, kv_capacity=w.max_seqlen)
        self.ws = torch.empty(H.workspace_bytes(self.shape), dtype=torch.uint8, device=dev)
        H.workspace_init(self.ws)
        self.resident = resident_layers
        self.q, self.K, self.V = [], [], []
        for l in range(w.layers):
            q, K, V = W.layer_inputs(w, l, device=dev, heads=heads)
            self.q.append(q)
            if l < resident_layers:
                self.K.append(K)
                self.V.append(V)
            else:
                del K, V
        torch.cuda.synchronize()
        self.Ks = [self.K[l % resident_layers] for l in range(w.layers)]
        self.Vs = [self.V[l % resident_layers] for l in range(w.layers)]
        self.outs = [torch.empty(w.batch, self.nq, w.head_dim, device=dev)
                     for _ in range(w.layers)]
        self.topk = torch.full((w.layers, w.batch, self.nkv, w.topk), -1,
                               dtype=torch.int32, device=dev)

    def full_bytes(self) -> int:
        """K+V bytes of one reset layer on this GPU."""
        return self.w.kv_bytes_per_layer() * self.nkv // self.w.num_kv_heads

    def reuse_bytes(self) -> int:
        """K+V bytes one reuse layer touches on this GPU."""
        return self.w.kv_bytes_reuse_layer() * self.nkv // self.w.num_kv_heads

    def step(self, policy, stream=None):
        L = len(policy)
        self.H.decode_step(self.shape, policy, self.q[:L], self.Ks[:L], self.Vs[:L],
                           self.seqlens, self.outs[:L], self.topk[:L], self.ws, stream=stream)

    def graph(self, policy):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.step(policy)  # warm (one-time host setup outside capture)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g, stream=s):
            self.step(policy, stream=torch.cuda.current_stream())
        g.kernel_nodes = graph_kernel_nodes(g)
        g.instantiate()
        torch.cuda.synchronize()
        return g


def graph_kernel_nodes(g) -> int:
    """Kernel launches one replay of a captured graph makes (counted from
    the graph's own node list, so every launch of the library is counted)."""
    from cuda.bindings import runtime as rt
    graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
    err, _, n = rt.cudaGraphGetNodes(graph, 0)
    assert err == rt.cudaError_t.cudaSuccess, err
    err, nodes, n = rt.cudaGraphGetNodes(graph, n)
    assert err == rt.cudaError_t.cudaSuccess, err
    kinds = [rt.cudaGraphNodeGetType(nd)[1] for nd in nodes[:n]]
    return sum(1 for k in kinds if k == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)


def policy_rule(args, w) -> str:
    if args.policy == "jump3":
        return "jump3 (reset every 3rd layer)"
    if w.policy is not None:
        return "fixed by the workload"
    theta = w.theta if args.theta is None else args.theta
    rule = f"dp theta={theta:g} profile_steps={max(1, args.profile_steps)}"
    if args.profile_seeds > 1:
        rule += f" profile_seeds={args.profile_seeds}"
    if args.token_topk > 0:
        rule += f" token_topk={args.token_topk}"
    return rule


def seed_variant(w: W.Workload, s: int) -> W.Workload:
    """Workload s of a multi-seed profiling run: the same shapes and lengths,
    its own salient structure and noise (s = 0: the benchmarked workload)."""
    return w if s == 0 else dataclasses.replace(w, seed=w.seed + 7919 * s)


def step_bytes(w: W.Workload, policy) -> int:
    """K+V bytes one hybrid step touches over the whole workload."""
    R = sum(policy)
    return R * w.kv_bytes_per_layer() + (w.layers - R) * w.kv_bytes_reuse_layer()


def parallelism(args, world: int) -> str:
    if args.shard == "heads":
        return f"kv-head shards x{world}"
    return f"sequence shards x{world} (each GPU its own batch of the workload)"


def config_of(w: W.Workload, policy, args, world: int) -> dict:
    """The workload as both arms name it (the same keys and values)."""
    return {
        "workload": workload_desc(w),
        "policy": "".join("R" if x else "U" for x in policy),
        "policy_rule": policy_rule(args, w),
        "resets": int(sum(policy)),
        "l2": "inputs larger than L2: a step streams %.2f GB" % (step_bytes(w, policy) / 1e9),
        "parallelism": parallelism(args, world),
    }


def profile_layer_sets(m: Model, H, q, K, V, token_topk: int) -> np.ndarray:
    """Index sets of one layer run as a reset layer, one per (sequence, KV
    head): its top-k blocks, or with token_topk > 0 its top-`token_topk`
    tokens (token scores on the GPU, selection on the host)."""
    w = m.w
    out = torch.empty(w.batch, m.nq, w.head_dim, device="cuda")
    tk = torch.empty(w.batch, m.nkv, w.topk, dtype=torch.int32, device="cuda")
    if token_topk <= 0:
        H.decode_full(m.shape, q, K, V, m.seqlens, out, tk, m.ws)
        return tk.cpu().numpy().reshape(w.batch * m.nkv, w.topk)
    scores = torch.empty(w.batch, m.nkv, max(1, w.max_seqlen), device="cuda")
    H.token_scores(m.shape, q, K, V, m.seqlens, out, tk, scores, m.ws)
    sc = scores.cpu().numpy().reshape(w.batch * m.nkv, -1)
    lengths = np.repeat(np.array(w.seqlens, dtype=np.int32), m.nkv)
    return H.token_topk(sc, token_topk, lengths)


def derive_policy(m: Model, H, rule: str = "dp", theta=None, profile_steps: int = 1,
                  profile_seeds: int = 1, token_topk: int = 0, pooled: bool = True):
    """The step's reset/reuse policy.

    dp: profiling run(s) with every layer full -> overlap matrix -> DP policy
    (HyLRA summary §2.2).  With profile_steps P > 1 the index sets of P decode
    steps (fresh queries, same cache) are pooled into one matrix; with
    profile_seeds S > 1 those of S workloads that differ only by seed; with
    token_topk > 0 the sets are top-k tokens instead of blocks.  Over several
    ranks the matrix is pooled from every rank's index sets (integer counts
    summed over ranks), so all ranks derive the single-GPU policy.  A
    workload with a fixed policy keeps it.  jump3: a reset every third layer
    (the static baseline of §4)."""
    w = m.w
    if rule == "jump3":
        pol, _ = H.static_policy(w.layers, 3)
        return pol, None
    if w.policy is not None:
        return tuple(w.policy), None
    allfull = (1,) * w.layers
    sets = []
    q0 = list(m.q)
    for p in range(max(1, profile_steps)):
        if p > 0:
            m.q = [W.step_query(w, l, p, device="cuda", heads=m.heads) for l in range(w.layers)]
        if token_topk > 0:
            sets.append(np.stack([profile_layer_sets(m, H, m.q[l], m.Ks[l], m.Vs[l], token_topk)
                                  for l in range(w.layers)]))
        else:
            m.step(allfull)  # the step's own launch configuration
            torch.cuda.synchronize()
            sets.append(m.topk.cpu().numpy().reshape(w.layers, w.batch * m.nkv, w.topk))
    m.q = q0
    for s in range(1, max(1, profile_seeds)):
        ws = seed_variant(w, s)
        per_layer = []
        for l in range(w.layers):
            q, K, V = W.layer_inputs(ws, l, device="cuda", heads=m.heads)
            per_layer.append(profile_layer_sets(m, H, q, K, V, token_topk))
            del q, K, V
        sets.append(np.stack(per_layer))
        torch.cuda.empty_cache()
    sets = np.concatenate(sets, axis=1)
    M = D.pooled_similarity(H, sets, device="cuda") if pooled else H.similarity(sets)
    pol, R, S = H.dp_policy(M, w.theta if theta is None else theta)
    return pol, M


def output_error_vs_full(m: Model, g_h, g_f):
    """Relative Frobenius error of each layer's hybrid output against full
    attention on the same inputs (a synthetic stand-in for the pages'
    accuracy comparison): (mean over reuse layers, max over layers)."""
    g_h.replay()
    torch.cuda.synchronize()
    oh = [o.clone() for o in m.outs]
    g_f.replay()
    torch.cuda.synchronize()
    errs = [float((a - b).norm() / b.norm().clamp_min(1e-30)) for a, b in zip(oh, m.outs)]
    return errs


def timed_replays(g, steps, dist_on):
    D.barrier()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        g.replay()
    e1.record(st)
    torch.cuda.synchronize()
    D.barrier()
    return e0.elapsed_time(e1) / steps


def max_over_ranks(x: float, dist_on: bool) -> float:
    return D.max_over_ranks(x, device="cuda") if dist_on else x


def e2e_step_time(m: Model, H, policy, steps, warmup, dist_on):
    """Through hylra_decode_step_host: q from pinned host memory, outputs back
    (every step: the q copy in, the step, the output and index copies out)."""
    w = m.w
    q_host = torch.stack([q.cpu() for q in m.q]).pin_memory()
    q_dev = torch.empty_like(q_host, device="cuda")
    out_dev = torch.empty(w.layers, w.batch, m.nq, w.head_dim, device="cuda")
    out_host = torch.empty(out_dev.shape, dtype=torch.float32).pin_memory()
    tk_dev = torch.full((w.layers, w.batch, m.nkv, w.topk), -1, dtype=torch.int32,
                        device="cuda")
    tk_host = torch.empty(tk_dev.shape, dtype=torch.int32).pin_memory()

    def call(stream=None):
        H.decode_step_host(m.shape, policy, q_host, q_dev, m.Ks, m.Vs, m.seqlens, out_dev,
                           out_host, tk_dev, tk_host, m.ws, stream=stream)

    # the call captured once into a CUDA graph (its copies included), as a
    # serving loop would replay it
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        call(stream=torch.cuda.current_stream())

    for _ in range(warmup):
        g.replay()
    ms = timed_replays(g, steps, dist_on)
    h2d = q_host.numel() * q_host.element_size()
    d2h = out_host.numel() * 4 + tk_host.numel() * 4
    del g
    return ms, h2d, d2h


def offload_measure(m: Model, H, policy, steps, warmup, dist_on):
    """Index-guided offloading (HyLRA summary §2.4): the reuse layers' caches
    move to pinned host memory and each reuse layer gathers only its reused
    blocks across the host link.  Times the graph-replayed step and, for
    reference, a plain host-to-device copy of the same bytes per step."""
    w = m.w
    offloaded = tuple(0 if x else 1 for x in policy)
    Ko, Vo = [], []
    for l in range(w.layers):
        if offloaded[l]:
            Ko.append(m.Ks[l].cpu().pin_memory())
            Vo.append(m.Vs[l].cpu().pin_memory())
        else:
            Ko.append(m.Ks[l])
            Vo.append(m.Vs[l])
    n = H.stage_bytes(m.shape)  # bytes of one slot = bf16 elements of the two slots
    Ks = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    Vs = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        H.decode_step_offload(m.shape, policy, m.q, Ko, Vo, offloaded, m.seqlens, m.outs, m.topk,
                              Ks, Vs, m.ws)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        H.decode_step_offload(m.shape, policy, m.q, Ko, Vo, offloaded, m.seqlens, m.outs, m.topk,
                              Ks, Vs, m.ws, stream=torch.cuda.current_stream())
    for _ in range(warmup):
        g.replay()
    ms = timed_replays(g, steps, dist_on)
    # bytes that cross the link per step: k' blocks of K and V per (b, h) per
    # offloaded layer
    host_bytes = m.reuse_bytes() * sum(offloaded)
    # a plain pinned-host-to-device copy of those bytes, for the link's rate
    src = torch.empty(host_bytes, dtype=torch.uint8).pin_memory()
    dst = torch.empty(host_bytes, dtype=torch.uint8, device="cuda")
    dst.copy_(src, non_blocking=True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(3):
        dst.copy_(src, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    copy_ms = e0.elapsed_time(e1) / 3
    del g
    return {"us_per_step": round(ms * 1000.0, 3),
            "offloaded_layers": int(sum(offloaded)),
            "host_link_bytes_per_step": int(host_bytes),
            "host_link_gbs": round(host_bytes / (ms * 1e-3) / 1e9, 1),
            "plain_copy_gbs": round(host_bytes / (copy_ms * 1e-3) / 1e9, 1),
            "device_cache_bytes_moved_to_host": int(m.full_bytes() * sum(offloaded))}


def oracle_sample_data(w: W.Workload, reset_layer, reuse_layer, head=0):
    """The inputs of the oracle's bounded sample, as fp64 host arrays: KV
    head `head` of every sequence (its query rows, keys and values) in one
    reset layer and one reuse layer.  reset_layer / reuse_layer: (q, K, V)
    tensors (any device) holding at least KV head `head`; reuse_layer may be
    None (a policy without reuse layers)."""
    r = w.group

    def prep(layer):
        q, K, V = layer
        out = []
        for b in range(w.batch):
            out.append((q[b, head * r:(head + 1) * r].double().cpu().numpy(),
                        W.per_sequence(w, K, b)[head:head + 1].double().cpu().numpy(),
                        W.per_sequence(w, V, b)[head:head + 1].double().cpu().numpy()))
        return out

    return head, prep(reset_layer), (prep(reuse_layer) if reuse_layer is not None else None)


def oracle_sample(w: W.Workload, data, policy):
    """Time the fp64 oracle, single-threaded, on a bounded sample of one
    decode step (oracle_sample_data): the sampled KV head of every sequence
    through one reset layer (full attention, block scores, top-k) and one
    reuse layer (attention over the blocks that reset layer selected).  A
    step is R reset and L - R reuse layers over all Hkv heads, so the two
    times scale to it exactly (the oracle's cost per layer does not depend on
    which layer it is).  Returns (seconds per step, sample text, threads)."""
    from oracle import hylra_oracle as O
    from threadpoolctl import threadpool_limits
    head, d_reset, d_reuse = data
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        idx = [O.full_layer(qb, kb, vb, w.seqlens[b], w.topk)[2]
               for b, (qb, kb, vb) in enumerate(d_reset)]
        t1 = time.perf_counter()
        if d_reuse is not None:
            for b, (qb, kb, vb) in enumerate(d_reuse):
                O.reuse_attention(qb, kb, vb, w.seqlens[b], idx[b])
        t2 = time.perf_counter()
    R = sum(policy)
    sec = w.num_kv_heads * (R * (t1 - t0) + (w.layers - R) * (t2 - t1))
    sample = (f"KV head {head} of every sequence through one reset and one reuse layer, "
              f"single-threaded; scaled to {w.num_kv_heads} KV heads x ({R} reset + "
              f"{w.layers - R} reuse layers)")
    return sec, sample, 1


def run_ours(args, rank, world, dist_on):
    from kv_cache_sparsity_b200 import hylra as H
    hbuild.build()
    H.load()
    w0 = W.config(args.config)
    if args.shard == "heads":
        w, heads = w0, D.shard(w0.num_kv_heads, rank, world)
        if len(heads) == 0:
            raise SystemExit(f"{world} ranks for {w0.num_kv_heads} KV heads: a rank would hold none")
    else:
        # rank r: its own batch of the global batch (rank 0: the configured workload)
        w, heads = seed_variant(w0, rank), range(w0.num_kv_heads)
    free = torch.cuda.mem_get_info()[0]
    per_layer = w.kv_bytes_per_layer() * len(heads) // w.num_kv_heads  # K and V on this GPU
    resident = w.layers
    if per_layer * w.layers > free * 0.85:
        resident = max(1, int(free * 0.85 // per_layer))
    m = Model(w, H, resident, heads)
    if args.shard == "heads":
        # every rank profiles its heads; the counts are pooled over the ranks
        policy, M = derive_policy(m, H, args.policy, args.theta, args.profile_steps,
                                  args.profile_seeds, args.token_topk)
    else:
        # the configured workload's policy (rank 0's), the same on every rank
        policy = None
        if rank == 0:
            policy, M = derive_policy(m, H, args.policy, args.theta, args.profile_steps,
                                      args.profile_seeds, args.token_topk, pooled=False)
        policy = D.broadcast_policy(policy, device="cuda")
    L = w.layers
    allfull = (1,) * L
    one_then_reuse = (1,) + (0,) * (L - 1)
    R = sum(policy)
    g_h = m.graph(policy)
    g_f = m.graph(allfull)
    g_u = m.graph(one_then_reuse)
    g_1 = m.graph((1,))
    for _ in range(args.warmup):
        for g in (g_h, g_f, g_u, g_1):
            g.replay()
    torch.cuda.synchronize()
    assert H.read_status(m.ws) == 0, "device status set during warm-up"

    uuid = str(getattr(torch.cuda.get_device_properties(0), "uuid", ""))
    if uuid and not uuid.startswith("GPU-"):
        uuid = "GPU-" + uuid
    clk = ClockSampler(uuid)
    clk.start()
    ms_h = timed_replays(g_h, args.steps, dist_on)
    ms_f = timed_replays(g_f, args.steps, dist_on)
    ms_u = timed_replays(g_u, args.steps, dist_on)
    ms_1 = timed_replays(g_1, args.steps, dist_on)
    # keep the GPU busy long enough for the sampler when the timed region is short
    fill = 0.0 if args.no_clock_fill else 0.6
    t_end = time.time() + max(0.0, fill - (ms_h + ms_f + ms_u + ms_1) * args.steps / 1000.0)
    while time.time() < t_end:
        g_h.replay()
        torch.cuda.synchronize()
    clocks = clk.stop()
    ms_h = max_over_ranks(ms_h, dist_on)
    ms_f = max_over_ranks(ms_f, dist_on)
    ms_u = max_over_ranks(ms_u, dist_on)
    ms_1 = max_over_ranks(ms_1, dist_on)
    status = H.read_status(m.ws)

    e2e_ms, h2d, d2h = e2e_step_time(m, H, policy, max(3, args.steps // 4), args.warmup,
                                     dist_on)
    e2e_ms = max_over_ranks(e2e_ms, dist_on)
    g_launches = g_h.kernel_nodes
    errs = output_error_vs_full(m, g_h, g_f)
    reuse_errs = [e for e, x in zip(errs, policy) if not x] or [0.0]
    del g_h, g_f, g_u, g_1
    offload = (offload_measure(m, H, policy, max(3, args.steps // 4), args.warmup, dist_on)
               if args.offload else None)

    peak, peak_kind = measured_hbm_peak()
    # the whole job: every rank's batch (sequence shards) or the one workload
    job_batches = world if args.shard == "batch" else 1
    job_bytes = step_bytes(w, policy) * job_batches
    us_h = ms_h * 1000.0
    kv_gbs = job_bytes / (ms_h * 1e-3) / 1e9
    full_b, reuse_b = m.full_bytes(), m.reuse_bytes()
    reset_us = ms_f * 1000.0 / L
    reuse_us = (ms_u - ms_1) * 1000.0 / max(1, L - 1)
    achieved = full_b / (reset_us * 1e-6) / 1e9

    def layer_rate(nbytes, us):
        gbs = nbytes / (us * 1e-6) / 1e9
        return {"us": round(us, 3), "kv_bytes": int(nbytes), "gbs": round(gbs, 1),
                "frac_of_measured": round(gbs / peak, 4),
                "frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4)}

    line = {
        "metric": METRIC,
        "value": round(us_h, 3),
        "unit": "us/step",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_h, 6),
        "higher_is_better": False,
        "scaling": "weak" if args.shard == "batch" else "strong",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded salient-block K, iid V; see workloads.py)",
        "config": config_of(w, policy, args, world),
        "kv_heads_per_gpu": len(heads),
        "resident_layer_caches": m.resident,
        "kv_bytes_per_step": job_bytes,
        "kv_gbs": round(kv_gbs, 1),
        "kv_frac_of_8tbs": round(kv_gbs / NOMINAL_HBM_GBS, 4),
        "full_us_per_step": round(ms_f * 1000.0, 3),
        "speedup_vs_full": round(ms_f / ms_h, 4),
        "sequences_per_s": round(job_batches * w.batch / (ms_h * 1e-3), 1),
        "reset_layer": layer_rate(full_b, reset_us),
        "reuse_layer": dict(layer_rate(reuse_b, reuse_us),
                            how="(one reset + %d reuse layers) - (one reset layer), per reuse "
                                "layer, graph-replayed" % (L - 1)),
        "roofline": {
            "bound": "hbm",
            "kernel": "reset layer (streaming + merge kernels, the step's dominant work)",
            "achieved": round(achieved, 1),
            "peak": peak,
            "peak_kind": peak_kind,
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": ncu_traffic("full_kernel", w.name),
            "algorithmic_bytes_per_launch": full_b,
            "avg_launch_us": round(reset_us, 3),
        },
        "e2e": {"value": round(e2e_ms * 1000.0, 3), "unit": "us/step",
                "how": "hylra_decode_step_host captured in a CUDA graph, copies included",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": g_launches * args.steps,
        "quality_vs_full": {"rel_err_mean_reuse_layers": round(statistics.mean(reuse_errs), 5),
                            "rel_err_max": round(max(errs), 5)},
        "offload": offload,
        "clocks": clocks,
        "device_status": status,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        first_reuse = next((l for l in range(L) if not policy[l]), None)
        data = oracle_sample_data(
            w, (m.q[0], m.Ks[0], m.Vs[0]),
            None if first_reuse is None else (m.q[first_reuse], m.Ks[first_reuse],
                                              m.Vs[first_reuse]))
        sec, sample, threads = oracle_sample(w, data, policy)
        line["cpu_baseline"] = {"value": round(sec * 1e6, 1), "unit": "us/step",
                                "cores": threads, "kind": "oracle", "sample": sample}
    return line


# ----------------------------------------------------------- reference arm

def oracle_policy(w: W.Workload, args, gen: str):
    """The policy the oracle derives from its own profiling run: every layer
    a reset layer (oracle.layer_topk on every layer, sequence and KV head),
    its overlap matrix, its DP.  Inputs are drawn layer by layer on `gen` and
    copied to the host."""
    from oracle import hylra_oracle as O
    if args.policy == "jump3":
        return O.static_policy(w.layers, 3)[0]
    if w.policy is not None:
        return tuple(w.policy)
    P = max(1, args.profile_steps)
    S = max(1, args.profile_seeds)
    Hkv = w.num_kv_heads
    k = args.token_topk if args.token_topk > 0 else w.topk
    rank_fn = O.layer_token_topk if args.token_topk > 0 else O.layer_topk
    sets = np.full((w.layers, (P + S - 1) * w.batch * Hkv, k), -1, dtype=np.int32)
    # the sets in our arm's order: steps 0..P-1 of the workload, then seeds 1..S-1
    runs = [(0, p) for p in range(P)] + [(s, 0) for s in range(1, S)]
    for l in range(w.layers):
        for j, (s, p) in enumerate(runs):
            ws = seed_variant(w, s)
            q, K, _ = W.layer_inputs(ws, l, device=gen)
            K = K.cpu()
            qp = (q if p == 0 else W.step_query(ws, l, p, device=gen)).cpu()
            for b in range(w.batch):
                _, tk = rank_fn(qp[b].double().numpy(), W.per_sequence(w, K, b).double().numpy(),
                                w.seqlens[b], k)
                sets[l, (j * w.batch + b) * Hkv:(j * w.batch + b + 1) * Hkv] = tk
            del q, K, qp
            if gen == "cuda":
                torch.cuda.empty_cache()
    M = O.similarity_matrix(sets)
    return O.dp_policy(M, w.theta if args.theta is None else args.theta)[0]


def run_reference(args, world):
    """The fp64 oracle, as it stands, on the host cores (no GPU needed; with
    one, only to draw the same inputs as our arm)."""
    w = W.config(args.config)
    # the same values as our arm: torch's generator differs between CPU and
    # GPU, so the inputs are drawn on the GPU when there is one (and only
    # then copied to the host, where all the timed work runs)
    gen = "cuda" if torch.cuda.is_available() else "cpu"
    policy = oracle_policy(w, args, gen)
    first_reuse = next((l for l in range(w.layers) if not policy[l]), None)
    data = oracle_sample_data(
        w, W.layer_inputs(w, 0, device=gen),
        W.layer_inputs(w, first_reuse, device=gen) if first_reuse is not None else None)
    if gen == "cuda":
        torch.cuda.empty_cache()
    for _ in range(args.warmup):
        oracle_sample(w, data, policy)
    times = []
    sample = ""
    threads = 1
    for _ in range(args.steps):
        sec, sample, threads = oracle_sample(w, data, policy)
        times.append(sec)
    us = statistics.mean(times) * 1e6
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(us, 1),
        "unit": "us/step",
        "n_gpus": 0,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(us / 1000.0, 3),
        "higher_is_better": False,
        "scaling": "weak" if args.shard == "batch" else "strong",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded salient-block K, iid V; see workloads.py)",
        "config": config_of(w, policy, args, world),
        "cpu_baseline": {"value": round(us, 1), "unit": "us/step", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(us, 1), "unit": "us/step", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# --------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="ragged16", choices=W.CONFIG_NAMES,
                    help="workload (default: the largest that fits one GPU)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--policy", default="dp", choices=["dp", "jump3"],
                    help="dp: profiled overlap matrix + DP (HyLRA); jump3: reset every 3rd layer")
    ap.add_argument("--theta", type=float, default=None,
                    help="DP threshold (default: the workload's, 0.8)")
    ap.add_argument("--offload", action="store_true",
                    help="also time the step with the reuse layers' caches in host memory")
    ap.add_argument("--profile-steps", type=int, default=1,
                    help="decode steps pooled into the profiled overlap matrix")
    ap.add_argument("--profile-seeds", type=int, default=1,
                    help="synthetic workloads (seeds) pooled into the profiled overlap matrix")
    ap.add_argument("--shard", default="batch", choices=["batch", "heads"],
                    help="N GPUs: batch = each GPU its own batch (weak), heads = KV heads of one "
                         "workload split over the GPUs (strong)")
    ap.add_argument("--token-topk", type=int, default=0,
                    help="profile top-k tokens (this many per head) instead of top-k blocks")
    ap.add_argument("--no-clock-fill", action="store_true",
                    help="skip the extra busy window for the clock sampler (profiler runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank, local, world = D.rank_env()

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return 0

    dist_on = world > 1
    torch.cuda.set_device(local)
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    line = run_ours(args, rank, world, dist_on)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
