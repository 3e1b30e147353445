"""Pins for the oracle's overlap matrix and DP policy (CPU only)."""

import json
import os

import numpy as np
import pytest

from oracle import hylra_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_similarity_hand_worked():
    g = _load("similarity_3layer.json")
    M = O.similarity_matrix(np.array(g["topk"]))
    assert M.tolist() == g["M"]


def test_similarity_identical_and_disjoint():
    a = np.array([[[0, 1, 2, 3]], [[3, 2, 1, 0]], [[4, 5, 6, 7]]])
    M = O.similarity_matrix(a)
    assert M[1, 0] == 1.0 and M[2, 0] == 0.0 and M[2, 1] == 0.0
    assert np.all(np.diag(M) == 1.0)
    assert np.all(np.triu(M, 1) == 0.0)


def test_similarity_padding_is_ignored():
    a = np.array([[[0, 1, -1, -1]], [[1, 5, -1, -1]]])
    M = O.similarity_matrix(a)
    assert M[1, 0] == 0.5 and M[1, 1] == 1.0


def _dyadic_matrix(L, rng, denom=64):
    M = np.zeros((L, L))
    for t in range(L):
        for s in range(t):
            M[t, s] = rng.integers(0, denom + 1) / denom
        M[t, t] = 1.0
    return M


@pytest.mark.parametrize("L", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("theta", [0.0, 0.25, 0.5, 0.8, 1.0])
def test_dp_matches_bruteforce(L, theta):
    rng = np.random.default_rng(L * 100 + int(theta * 100))
    for _ in range(25):
        M = _dyadic_matrix(L, rng)
        assert O.dp_policy(M, theta) == O.dp_policy_bruteforce(M, theta)


def test_dp_hand_worked():
    g = _load("dp_4layer.json")
    M = np.array(g["M"])
    for case in g["cases"]:
        pol, R, S = O.dp_policy(M, case["theta"])
        assert list(pol) == case["policy"]
        assert R == case["resets"]
        assert S == case["sim"]


def test_dp_closed_forms():
    rng = np.random.default_rng(7)
    for L in (4, 9, 16, 32):
        M = _dyadic_matrix(L, rng)
        # theta >= 1: no similarity can exceed it -> every layer resets
        pol, R, S = O.dp_policy(M, 1.0)
        assert pol == (1,) * L and R == L and S == 0.0
        # theta below every entry: one reset; the best source is layer 0 or a
        # later reset, but a single reset already minimises -> sim = sum M[j][0]
        pol, R, S = O.dp_policy(M, -1.0)
        assert R == 1 and pol == (1,) + (0,) * (L - 1)
        assert S == sum(M[j, 0] for j in range(1, L))


def test_dp_resets_monotone_in_theta():
    rng = np.random.default_rng(11)
    M = _dyadic_matrix(12, rng)
    last = 0
    for theta in np.linspace(-0.1, 1.0, 23):
        _, R, _ = O.dp_policy(M, theta)
        assert R >= last
        last = R


def test_dp_strict_threshold():
    M = np.array([[1.0, 0.0], [0.5, 1.0]])
    assert O.dp_policy(M, 0.5)[0] == (1, 1)     # 0.5 does not exceed 0.5
    assert O.dp_policy(M, 0.4999)[0] == (1, 0)


@pytest.mark.parametrize("L,period", [(1, 3), (2, 3), (3, 3), (4, 3), (10, 3), (32, 3), (9, 1),
                                      (6, 6), (6, 100)])
def test_static_policy_closed_form(L, period):
    """A reset at layers 0, period, 2 period, ...: ceil(L / period) resets."""
    pol, R = O.static_policy(L, period)
    assert len(pol) == L and pol[0] == O.RESET
    assert R == -(-L // period) == sum(pol)
    assert [i for i, x in enumerate(pol) if x == O.RESET] == list(range(0, L, period))


def test_overlap_counts_hand_worked():
    g = _load("similarity_3layer.json")
    inter, total = O.overlap_counts(np.array(g["topk"]))
    assert inter.tolist() == g["inter"] and total.tolist() == g["total"]
    assert O.similarity_from_counts(inter, total).tolist() == g["M"]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_overlap_counts_add_over_disjoint_groups_of_sets(seed):
    """Counts of two disjoint groups of index sets add up to the counts of
    all of them, and the ratio of the sums is the pooled matrix exactly."""
    rng = np.random.default_rng(seed)
    L, S, k, nb = 6, 10, 5, 12
    topk = np.full((L, S, k), -1, dtype=np.int32)
    for l in range(L):
        for u in range(S):
            m = int(rng.integers(0, k + 1))
            topk[l, u, :m] = rng.choice(nb, size=m, replace=False)
    i_all, t_all = O.overlap_counts(topk)
    cut = int(rng.integers(1, S))
    i_a, t_a = O.overlap_counts(topk[:, :cut])
    i_b, t_b = O.overlap_counts(topk[:, cut:])
    assert np.array_equal(i_a + i_b, i_all) and np.array_equal(t_a + t_b, t_all)
    M = O.similarity_from_counts(i_a + i_b, t_a + t_b)
    assert M.tobytes() == O.similarity_matrix(topk).tobytes()
    # brute force on the definition: one set at a time
    for t in range(L):
        assert t_all[t] == sum(int((topk[t, u] >= 0).sum()) for u in range(S))
        for s in range(t + 1):
            brute = sum(len(set(topk[s, u][topk[s, u] >= 0]) & set(topk[t, u][topk[t, u] >= 0]))
                        for u in range(S))
            assert i_all[t, s] == brute
