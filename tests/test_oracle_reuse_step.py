"""Pins for the oracle's reuse attention and the per-step layer walk (CPU only)."""

import math

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

from oracle import hylra_oracle as O


def _sdpa_rows(q_g, K_rows, V_rows):
    qt = torch.from_numpy(q_g)[None, None, None, :]
    kt = torch.from_numpy(np.ascontiguousarray(K_rows))[None, None]
    vt = torch.from_numpy(np.ascontiguousarray(V_rows))[None, None]
    return F.scaled_dot_product_attention(qt, kt, vt)[0, 0, 0].numpy()


@pytest.mark.parametrize("n", [128, 700, 1025])
def test_reuse_with_every_block_equals_full(n):
    rng = np.random.default_rng(n)
    q = rng.standard_normal((8, 64))
    K = rng.standard_normal((2, n, 64))
    V = rng.standard_normal((2, n, 64))
    nb = O.num_blocks(n)
    idx = np.stack([rng.permutation(nb), rng.permutation(nb)])
    full, _ = O.full_attention(q, K, V, n)
    reuse = O.reuse_attention(q, K, V, n, idx)
    np.testing.assert_allclose(reuse, full, rtol=1e-12, atol=1e-13)


def test_reuse_subset_matches_sdpa_on_gathered_tokens():
    n, d = 1000, 32        # last block (7) holds 104 tokens
    rng = np.random.default_rng(4)
    q = rng.standard_normal((6, d))
    K = rng.standard_normal((3, n, d))
    V = rng.standard_normal((3, n, d))
    idx = np.array([[7, 2, -1], [0, -1, -1], [5, 6, 1]])
    out = O.reuse_attention(q, K, V, n, idx)
    for g in range(6):
        h = g // 2
        toks = []
        for b in idx[h]:
            if b >= 0:
                toks += list(range(128 * b, min(128 * b + 128, n)))
        ref = _sdpa_rows(q[g], K[h, toks], V[h, toks])
        np.testing.assert_allclose(out[g], ref, rtol=1e-12, atol=1e-13)


def test_reuse_empty_selection_is_zero():
    q = np.ones((2, 8))
    K = np.ones((1, 300, 8))
    V = np.ones((1, 300, 8))
    out = O.reuse_attention(q, K, V, 300, np.array([[-1, -1]]))
    assert np.all(out == 0.0)


def _block_world(n, d, logits_per_block, vals_per_block):
    """One KV head whose keys/values are constant per block.

    q = e0 * sqrt(d); key of block b = logit_b * e0, so every token of block b
    has logit logit_b exactly; value of block b = vals_per_block[b] * ones.
    """
    nb = O.num_blocks(n)
    q = np.zeros((1, d))
    q[0, 0] = math.sqrt(d)
    K = np.zeros((1, n, d))
    V = np.zeros((1, n, d))
    for b in range(nb):
        lo, hi = 128 * b, min(128 * b + 128, n)
        K[0, lo:hi, 0] = logits_per_block[b]
        V[0, lo:hi, :] = vals_per_block[b]
    return q, K, V


def test_step_reuse_layer_uses_last_reset_layers_blocks():
    """Closed form: layer 0 favours blocks {1, 3}; layer 1 (reuse) favours
    {0, 2} itself but must attend over {1, 3}; layer 2 resets and picks its
    own {0, 2}; layer 3 reuses {0, 2}."""
    n, d, k = 512, 8, 2
    vals = np.array([10.0, 20.0, 30.0, 40.0])
    hi_odd = np.array([0.0, 5.0, 0.0, 4.0])
    hi_even = np.array([3.0, 0.0, 2.0, 0.0])
    layers = []
    for lg in (hi_odd, hi_even, hi_even, hi_odd):
        q, K, V = _block_world(n, d, lg, vals)
        layers.append((q[None], K[None], V[None]))
    policy = (O.RESET, O.REUSE, O.RESET, O.REUSE)
    outs, topks = O.decode_step(policy, layers, [n], k)
    assert list(topks[0][0, 0]) == [1, 3]
    assert list(topks[1][0, 0]) == [1, 3]
    assert list(topks[2][0, 0]) == [0, 2]
    assert list(topks[3][0, 0]) == [0, 2]

    def closed(lg, blocks):
        w = scipy.special.softmax(lg[blocks])    # equal token counts per block
        return float(np.dot(w, vals[blocks]))

    full0 = float(np.dot(scipy.special.softmax(hi_odd), vals))
    assert outs[0][0, 0, 0] == pytest.approx(full0, rel=1e-13)
    assert outs[1][0, 0, 0] == pytest.approx(closed(hi_even, [1, 3]), rel=1e-13)
    assert outs[3][0, 0, 0] == pytest.approx(closed(hi_odd, [0, 2]), rel=1e-13)


def test_step_with_all_blocks_selected_matches_all_full():
    rng = np.random.default_rng(9)
    n, d, L = 600, 16, 4
    nb = O.num_blocks(n)
    layers = [(rng.standard_normal((2, 4, d)), rng.standard_normal((2, 2, n, d)),
               rng.standard_normal((2, 2, n, d))) for _ in range(L)]
    seqlens = [n, 300]
    outs_h, _ = O.decode_step((1, 0, 0, 1), layers, seqlens, nb)
    outs_f, _ = O.decode_step((1, 1, 1, 1), layers, seqlens, nb)
    for a, b in zip(outs_h, outs_f):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_step_rejects_leading_reuse():
    with pytest.raises(ValueError):
        O.decode_step((0, 1), [None, None], [1], 1)
