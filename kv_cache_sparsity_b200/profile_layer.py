"""Run one layer's decode kernels of a named workload, for profiling.

    python -m kv_cache_sparsity_b200.profile_layer --config llama8b_32k --kernel full --iters 3

Generates layer 0 (and layer 1 for the reuse kernel) of the workload on the
GPU, then launches the chosen kernel ``--warmup`` + ``--iters`` times with an
L2 flush (a 512 MB write) between launches, and prints the mean device time
of the timed launches.  Meant to be wrapped by a profiler (one small capture)
or run alone for a quick per-kernel timing.
"""

from __future__ import annotations

import argparse

import torch

from . import build as _build
from . import hylra as H
from . import workloads as W


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="llama8b_32k", choices=W.CONFIG_NAMES)
    ap.add_argument("--kernel", default="full", choices=["full", "reuse"])
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=2)
    args = ap.parse_args(argv)

    _build.build()
    w = W.config(args.config)
    dev = "cuda"
    seqlens = torch.tensor(w.seqlens, dtype=torch.int32, device=dev)
    offs = (torch.tensor(W.seq_offsets(w)[:-1], dtype=torch.int64, device=dev)
            if w.packed else None)
    dtype = H.BF16 if w.dtype == "bf16" else H.FP32
    if w.packed:
        shape = H.make_shape(w.batch, w.num_q_heads, w.num_kv_heads, w.topk, w.max_seqlen,
                             dtype=dtype, total_tokens=w.total_tokens, seq_offsets=offs)
    else:
        shape = H.make_shape(w.batch, w.num_q_heads, w.num_kv_heads, w.topk, w.max_seqlen,
                             dtype=dtype, kv_capacity=w.max_seqlen)
    ws = torch.empty(H.workspace_bytes(shape), dtype=torch.uint8, device=dev)
    H.workspace_init(ws)
    q0, K0, V0 = W.layer_inputs(w, 0, device=dev)
    out = torch.empty(w.batch, w.num_q_heads, w.head_dim, device=dev)
    topk = torch.empty(w.batch, w.num_kv_heads, w.topk, dtype=torch.int32, device=dev)
    H.decode_full(shape, q0, K0, V0, seqlens, out, topk, ws)
    if args.kernel == "reuse":
        q1, K1, V1 = W.layer_inputs(w, 1, device=dev)
        del K0, V0

        def run():
            H.decode_reuse(shape, q1, K1, V1, seqlens, topk, out, ws)
    else:
        def run():
            H.decode_full(shape, q0, K0, V0, seqlens, out, topk, ws)

    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    times = []
    for i in range(args.warmup + args.iters):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1) * 1000.0)
    assert H.read_status(ws) == 0
    print(f"{args.config} {args.kernel}: mean {sum(times) / len(times):.2f} us over "
          f"{len(times)} launches")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
