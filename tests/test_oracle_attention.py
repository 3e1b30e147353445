"""Pins for the oracle's attention, block scores and top-k (CPU only).

Each check ties the oracle to something other than itself: torch's fp64
scaled_dot_product_attention (a library routine), closed forms for
structured inputs, invariants of softmax, and hand-worked rankings.
"""

import math

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

from oracle import hylra_oracle as O


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, K, V):
    """torch SDPA, fp64, GQA with q-head g -> KV head g // r (the common convention)."""
    qt = torch.from_numpy(q)[None, :, None, :]
    kt = torch.from_numpy(np.ascontiguousarray(K))[None]
    vt = torch.from_numpy(np.ascontiguousarray(V))[None]
    return F.scaled_dot_product_attention(qt, kt, vt, enable_gqa=True)[0, :, 0, :].numpy()


@pytest.mark.parametrize("d,n,hq,hkv", [(4, 1, 2, 1), (16, 5, 8, 2), (128, 127, 8, 2),
                                        (128, 128, 4, 4), (32, 300, 8, 1), (128, 513, 32, 8)])
def test_full_attention_matches_sdpa(d, n, hq, hkv):
    q = _rand((hq, d), 1 + n)
    K = _rand((hkv, n + 3, d), 2 + n)
    V = _rand((hkv, n + 3, d), 3 + n)
    out, probs = O.full_attention(q, K, V, n)
    ref = _sdpa(q, K[:, :n], V[:, :n])
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(probs.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def test_single_token_returns_its_value():
    q = _rand((8, 128), 5)
    K = _rand((2, 4, 128), 6)
    V = _rand((2, 4, 128), 7)
    out, _ = O.full_attention(q, K, V, 1)
    for g in range(8):
        np.testing.assert_allclose(out[g], V[g // 4, 0], rtol=0, atol=0)


def test_equal_keys_average_values():
    n = 200
    q = _rand((4, 16), 8)
    K = np.repeat(_rand((1, 1, 16), 9), n, axis=1)
    V = _rand((1, n, 16), 10)
    out, _ = O.full_attention(q, K, V, n)
    np.testing.assert_allclose(out, np.repeat(V[0].mean(axis=0)[None], 4, axis=0),
                               rtol=1e-12, atol=1e-12)


def test_dominant_key_selects_its_value():
    d, n = 64, 50
    q = np.zeros((1, d))
    q[0, 0] = 1.0
    K = np.zeros((1, n, d))
    K[0, 17, 0] = 60.0 * math.sqrt(d)   # logit 60 vs 0
    V = _rand((1, n, d), 11)
    out, _ = O.full_attention(q, K, V, n)
    np.testing.assert_allclose(out[0], V[0, 17], rtol=0, atol=1e-20)


def test_gqa_grouping_is_contiguous():
    # q-heads 0..3 must read KV head 0, 4..7 KV head 1: make the heads differ
    d, n = 8, 3
    q = np.zeros((8, d))
    K = np.zeros((2, n, d))
    V = np.zeros((2, n, d))
    V[0] = 1.0
    V[1] = 2.0
    out, _ = O.full_attention(q, K, V, n)
    assert np.all(out[:4] == 1.0) and np.all(out[4:] == 2.0)


# ---------------------------------------------------------------- block scores

@pytest.mark.parametrize("n", [1, 127, 128, 129, 1000, 4096])
def test_block_scores_sum_to_group_size(n):
    q = _rand((8, 32), 12)
    K = _rand((2, n, 32), 13)
    V = _rand((2, n, 32), 14)
    _, probs = O.full_attention(q, K, V, n)
    S = O.block_scores(probs, 2)
    assert S.shape == (2, O.num_blocks(n))
    np.testing.assert_allclose(S.sum(axis=1), 4.0, rtol=0, atol=1e-11)


@pytest.mark.parametrize("n", [300, 384, 129])
def test_block_scores_closed_form_constant_block_keys(n):
    """Keys constant inside a block: block mass = softmax over blocks of
    (logit + log #tokens), summed over the group (a closed form)."""
    d, hq, hkv = 16, 6, 2
    r = hq // hkv
    nb = O.num_blocks(n)
    rng = np.random.default_rng(n)
    q = rng.standard_normal((hq, d))
    blockkeys = rng.standard_normal((hkv, nb, d))
    K = np.repeat(blockkeys, 128, axis=1)[:, :n]
    V = rng.standard_normal((hkv, n, d))
    _, probs = O.full_attention(q, K, V, n)
    S = O.block_scores(probs, hkv)
    counts = np.array([min(128, n - 128 * b) for b in range(nb)], dtype=np.float64)
    for h in range(hkv):
        expect = np.zeros(nb)
        for g in range(h * r, (h + 1) * r):
            lb = blockkeys[h] @ q[g] / math.sqrt(d)
            expect += scipy.special.softmax(lb + np.log(counts))
        np.testing.assert_allclose(S[h], expect, rtol=1e-12, atol=1e-14)


def test_fp32_rounding_is_round_to_nearest_even():
    one = 1.0
    half_ulp = 2.0 ** -24
    x = np.array([one + half_ulp, one + 3 * half_ulp, one + 1.5 * half_ulp])
    y = O.round_scores_fp32(x)
    assert y.dtype == np.float32
    assert float(y[0]) == 1.0                      # tie -> even (1.0)
    assert float(y[1]) == 1.0 + 2.0 ** -22         # tie -> even (1 + 2 ulp)
    assert float(y[2]) == 1.0 + 2.0 ** -23         # above half -> up


# ---------------------------------------------------------------------- top-k

def test_topk_all_equal_gives_lowest_indices():
    S = np.full(10, 0.5, dtype=np.float32)
    assert list(O.topk_blocks(S, 4)) == [0, 1, 2, 3]


def test_topk_monotone_inputs():
    S = np.arange(10, 0, -1).astype(np.float32)
    assert list(O.topk_blocks(S, 3)) == [0, 1, 2]
    S = np.arange(1, 11).astype(np.float32)
    assert list(O.topk_blocks(S, 3)) == [9, 8, 7]


def test_topk_permutation_inverse():
    rng = np.random.default_rng(3)
    perm = rng.permutation(50)
    S = np.empty(50, dtype=np.float32)
    S[perm] = np.arange(50, 0, -1)      # block perm[i] has rank i
    assert list(O.topk_blocks(S, 50)) == list(perm)


def test_topk_ties_hand_worked():
    S = np.array([3, 5, 5, 1, 5], dtype=np.float32)
    assert list(O.topk_blocks(S, 3)) == [1, 2, 4]
    assert list(O.topk_blocks(S, 4)) == [1, 2, 4, 0]


def test_topk_pads_when_fewer_blocks():
    S = np.array([0.25, 0.75], dtype=np.float32)
    assert list(O.topk_blocks(S, 4)) == [1, 0, -1, -1]


def test_topk_compares_in_fp32():
    # distinct in fp64 but equal after rounding to fp32 -> index order decides
    a = 0.3
    b = a + 1e-12
    S = O.round_scores_fp32(np.array([a, b]))
    assert S[0] == S[1]
    assert list(O.topk_blocks(S, 1)) == [0]


def test_topk_gap_certificate():
    S = np.array([4.0, 3.0, 2.0, 1.0], dtype=np.float32)
    assert O.topk_gap(S, 2) == pytest.approx(0.25)   # min((4-3)/4, (3-2)/3)
    assert O.topk_gap(np.array([1.0], dtype=np.float32), 4) == math.inf


# ------------------------------------------------------ ranking without output

@pytest.mark.parametrize("n,hq,hkv", [(0, 4, 2), (1, 4, 1), (300, 8, 2), (1000, 8, 8),
                                      (2049, 16, 4)])
def test_layer_topk_equals_full_layer_ranking(n, hq, hkv):
    """layer_topk (no V read) gives exactly full_layer's scores and indices."""
    rng = np.random.default_rng(n + 7 * hq)
    q = rng.standard_normal((hq, 64))
    K = rng.standard_normal((hkv, max(n, 1), 64))
    V = rng.standard_normal((hkv, max(n, 1), 64))
    _, S_full, tk_full = O.full_layer(q, K, V, n, 5)
    S, tk = O.layer_topk(q, K, n, 5)
    assert S.dtype == np.float32 and S.tobytes() == S_full.tobytes()
    assert np.array_equal(tk, tk_full)


def test_layer_topk_dominant_keys_rank_their_blocks_first():
    """One key per chosen block aligned with the query dominates: those
    blocks come first, in decreasing order of their logit bump."""
    d, n = 32, 128 * 10
    q = np.zeros((2, d))
    q[:, 0] = math.sqrt(d)
    K = np.zeros((1, n, d))
    for beta, bump in ((7, 30.0), (2, 25.0), (9, 20.0)):
        K[0, beta * 128 + 5, 0] = bump   # logit = bump on that one token
    _, tk = O.layer_topk(q, K, n, 3)
    assert list(tk[0]) == [7, 2, 9]


# ---------------------------------------------------------- token-level top-k

@pytest.mark.parametrize("n", [1, 5, 300, 1024])
def test_token_scores_sum_to_group_size_and_match_block_sums(n):
    q = _rand((8, 32), 21)
    K = _rand((2, n, 32), 22)
    V = _rand((2, n, 32), 23)
    _, probs = O.full_attention(q, K, V, n)
    St = O.token_scores(probs, 2)
    np.testing.assert_allclose(St.sum(axis=1), 4.0, rtol=0, atol=1e-11)
    Sb = O.block_scores(probs, 2)
    for beta in range(O.num_blocks(n)):
        lo, hi = 128 * beta, min(128 * beta + 128, n)
        np.testing.assert_allclose(St[:, lo:hi].sum(axis=1), Sb[:, beta], rtol=1e-13, atol=0)


def test_token_topk_hand_worked():
    """One KV head, two q-heads, five tokens; query along axis 0, keys with
    logits ln(1), ln(4), ln(2), ln(4), ln(3) for both heads: masses
    proportional to 1, 4, 2, 4, 3 (the two 4s tie: lower index first)."""
    d = 4
    q = np.zeros((2, d))
    q[:, 0] = math.sqrt(d)
    K = np.zeros((1, 5, d))
    K[0, :, 0] = np.log([1.0, 4.0, 2.0, 4.0, 3.0])
    S32, tk = O.layer_token_topk(q, K, 5, 3)
    np.testing.assert_allclose(S32[0], 2 * np.array([1, 4, 2, 4, 3]) / 14, rtol=1e-6)
    assert list(tk[0]) == [1, 3, 4]
    _, tk6 = O.layer_token_topk(q, K, 5, 6)
    assert list(tk6[0]) == [1, 3, 4, 2, 0, -1]


def test_token_topk_reduces_to_blocks_for_block_constant_keys():
    """Keys constant inside each 128-token block: every token of a block has
    the same score, so the top k*128 tokens are exactly the tokens of the top
    k blocks, and the token-level overlap matrix equals the block-level one."""
    d, hq, hkv, nb, k = 16, 4, 2, 12, 3
    rng = np.random.default_rng(5)
    sets_b, sets_t = [], []
    for layer in range(4):
        q = rng.standard_normal((hq, d))
        blockkeys = rng.standard_normal((hkv, nb, d)) * 2.0
        K = np.repeat(blockkeys, 128, axis=1)
        _, tkb = O.layer_topk(q, K, 128 * nb, k)
        _, tkt = O.layer_token_topk(q, K, 128 * nb, 128 * k)
        for h in range(hkv):
            want = sorted(t for beta in tkb[h] for t in range(128 * beta, 128 * beta + 128))
            assert sorted(tkt[h].tolist()) == want
        sets_b.append(tkb)
        sets_t.append(tkt)
    Mb = O.similarity_matrix(np.array(sets_b))
    Mt = O.similarity_matrix(np.array(sets_t))
    assert Mt.tobytes() == Mb.tobytes()
