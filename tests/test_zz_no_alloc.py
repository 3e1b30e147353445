"""hylra_decode_full_noalloc: the reset-layer call for callers that cannot
allocate device memory when they call (it runs on scratch compiled into the
library instead of a caller-supplied workspace).  Its results must match
hylra_decode_full's on the same inputs, on two calls in a row (the scratch
keeps the previous call's contents, so the second call checks that the call
clears what must start at zero).  This file is collected last on purpose."""

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


@pytest.mark.parametrize("w", [
    W.custom("noalloc_dense", batch=2, seqlens=(5000, 1300), num_q_heads=32, num_kv_heads=8,
             topk=16, seed=31),
    W.custom("noalloc_packed", batch=3, seqlens=(700, 4096, 129), num_q_heads=8,
             num_kv_heads=2, topk=8, packed=True, seed=32),
], ids=lambda w: w.name)
def test_noalloc_matches_workspace_call_twice(w):
    run = T.Runner(w)
    q, K, V = (t.cuda() for t in W.layer_inputs(w, 0, "cpu"))
    ref_out, ref_tk = run.full(q, K, V)
    assert run.status() == 0
    status = torch.full((1,), 0xFFFF, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out, tk = run.new_out(), run.new_topk()
        H.decode_full_noalloc(run.shape, q, K, V, run.seqlens, out, tk, status_out=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        T.check_out(out.cpu().numpy(), ref_out.cpu().numpy().astype("float64"), "bf16",
                    f"{w.name} noalloc")
        assert torch.equal(tk, ref_tk)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 1024 sequences x 8 KV heads x 2048 blocks of block records need far more
    # than the 8 MiB scratch; the call must refuse before launching anything
    offs = torch.zeros(1024, dtype=torch.int64, device="cuda")
    shape = H.make_shape(1024, 8, 8, 8, 262144, total_tokens=1, seq_offsets=offs)
    assert H.workspace_bytes(shape) > (8 << 20)
    dummy = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.HylraError) as e:
        H.decode_full_noalloc(shape, dummy, dummy, dummy,
                              torch.zeros(1024, dtype=torch.int32, device="cuda"),
                              torch.empty(16, device="cuda"),
                              torch.empty(16, dtype=torch.int32, device="cuda"))
    assert e.value.code == -4
