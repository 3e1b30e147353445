"""The benchmark's JSON contract, checked on the CPU through its reference
arm (the fp64 oracle timed on the host cores) on the small configuration."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    res = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
         "--steps", "1", "--warmup", "3"],
        capture_output=True, text=True, timeout=600, cwd=ROOT,
        env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout[-2000:]
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["steps"] == 1 and d["warmup"] == 3
    assert d["higher_is_better"] is False and d["unit"] == "us/step"
    assert d["value"] > 0 and d["ms_per_step"] == pytest.approx(d["value"] / 1000, rel=1e-3)
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert "workload" in d["config"]


def test_algorithmic_bytes_follow_the_shapes():
    """The roofline's algorithmic bytes: K and V (bf16, d = 128) of every
    cached token of every KV head for a reset layer, of the k' selected
    128-token blocks per head for a reuse layer; a step adds them by policy."""
    sys.path.insert(0, ROOT)
    import argparse
    import bench
    from kv_cache_sparsity_b200 import workloads as W
    kv = 2 * 2 * 128  # K and V, bf16, per token and KV head
    expect = {
        "llama8b_32k": (8 * 32768 * kv, 8 * 16 * 128 * kv),
        "llama8b_b8_64k": (8 * 8 * 65536 * kv, 8 * 8 * 32 * 128 * kv),
        "llama8b_128k": (8 * 131072 * kv, 8 * 64 * 128 * kv),
    }
    for name, (full, reuse) in expect.items():
        w = W.config(name)
        assert w.kv_bytes_per_layer() == full, name
        assert w.kv_bytes_reuse_layer() == reuse, name
    w = W.config("ragged16")
    assert w.kv_bytes_per_layer() == 8 * sum(w.seqlens) * kv
    assert min(w.seqlens) >= 32 * 128  # every sequence has k = 32 blocks to reuse
    assert w.kv_bytes_reuse_layer() == 16 * 8 * 32 * 128 * kv
    policy = (1, 0, 0, 1) + (0,) * (w.layers - 4)
    assert bench.step_bytes(w, policy) == 2 * w.kv_bytes_per_layer() + (w.layers - 2) * \
        w.kv_bytes_reuse_layer()
    args = argparse.Namespace(policy="dp", theta=None, profile_steps=1, profile_seeds=1,
                              token_topk=0, shard="batch")
    cfg = bench.config_of(w, policy, args, 1)
    assert cfg["policy"] == "RUUR" + "U" * (w.layers - 4) and cfg["resets"] == 2
    assert set(cfg) == {"workload", "policy", "policy_rule", "resets", "l2", "parallelism"}


def test_seed_variant_keeps_shapes_and_changes_the_draw():
    sys.path.insert(0, ROOT)
    import bench
    from kv_cache_sparsity_b200 import workloads as W
    w = W.config("ragged16")
    assert bench.seed_variant(w, 0) is w
    v = bench.seed_variant(w, 3)
    assert v.seed != w.seed and v.seqlens == w.seqlens and v.layers == w.layers
    assert (v.num_q_heads, v.num_kv_heads, v.topk) == (w.num_q_heads, w.num_kv_heads, w.topk)
