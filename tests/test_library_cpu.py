"""C-ABI library checks that need no GPU: it loads, exports every symbol of
include/hylra.h, validates arguments on the host, and its host-side policy
functions (overlap matrix, DP) agree bit for bit with the oracle."""

import ctypes
import json
import os
import re

import numpy as np
import pytest

from kv_cache_sparsity_b200 import build as hbuild
from kv_cache_sparsity_b200 import hylra as H
from oracle import hylra_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    hbuild.build()
    return H.load()


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(hylra_\w+)\s*\(", text,
                                    re.MULTILINE))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert {"hylra_decode_full", "hylra_decode_reuse", "hylra_similarity",
            "hylra_dp_policy"} <= names
    for n in sorted(names):
        assert hasattr(lib, n), n
    assert set(H.EXPORTS) <= names


def test_version_and_strerror(lib):
    assert H.version() == 100
    assert H.strerror(0) == "ok"
    assert "workspace" in H.strerror(-4)


def _shape(**kw):
    base = dict(batch=1, num_q_heads=32, num_kv_heads=8, topk=16, max_seqlen=4096,
                kv_capacity=4096)
    base.update(kw)
    return H.make_shape(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=64), -2), (dict(block_size=64), -2), (dict(num_q_heads=30), -1),
    (dict(num_q_heads=80, num_kv_heads=8), -2), (dict(topk=0), -1), (dict(topk=5000), -2),
    (dict(max_seqlen=-1), -1), (dict(max_seqlen=300000, kv_capacity=300000), -2),
    (dict(kv_capacity=100), -1), (dict(batch=0), -1), (dict(batch=2000), -2),
    (dict(dtype=7), -1), (dict(kv_capacity=0, total_tokens=100), -1),
])
def test_shape_validation_before_any_device_call(lib, kw, code):
    n = ctypes.c_size_t(0)
    rc = lib.hylra_workspace_bytes(ctypes.byref(_shape(**kw)), ctypes.byref(n))
    assert rc == code


def test_null_pointers_rejected(lib):
    sh = _shape()
    rc = lib.hylra_decode_full(ctypes.byref(sh), None, None, None, None, None, None, None, 0, None)
    assert rc == -1
    rc = lib.hylra_dp_policy(0, None, 0.5, None, None, None)
    assert rc == -1


def test_step_rejects_leading_reuse_before_launch(lib):
    sh = _shape()
    pol = (ctypes.c_uint8 * 2)(0, 1)
    fake = (ctypes.c_void_p * 2)(16, 16)
    rc = lib.hylra_decode_step(ctypes.byref(sh), 2, pol, fake, fake, fake, 16, fake, 16, 256,
                               1 << 20, None)
    assert rc == -1


# ------------------------------------------------------- host policy parity

def test_similarity_golden(lib):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "similarity_3layer.json")))
    M = H.similarity(np.array(g["topk"]))
    assert M.tolist() == g["M"]


@pytest.mark.parametrize("seed", range(6))
def test_similarity_matches_oracle_bitwise(lib, seed):
    rng = np.random.default_rng(seed)
    L, S, k = int(rng.integers(1, 12)), int(rng.integers(1, 20)), int(rng.integers(1, 9))
    nb = int(rng.integers(k, 3 * k + 2))
    topk = np.full((L, S, k), -1, dtype=np.int32)
    for l in range(L):
        for u in range(S):
            kp = int(rng.integers(0, k + 1)) if seed % 2 else k
            topk[l, u, :kp] = rng.permutation(nb)[:kp]
    M = H.similarity(topk)
    Mo = O.similarity_matrix(topk)
    assert M.tobytes() == Mo.tobytes()


@pytest.mark.parametrize("seed", range(4))
def test_overlap_counts_match_oracle(lib, seed):
    rng = np.random.default_rng(50 + seed)
    L, S, k = int(rng.integers(1, 10)), int(rng.integers(1, 16)), int(rng.integers(1, 9))
    nb = int(rng.integers(k, 3 * k + 2))
    topk = np.full((L, S, k), -1, dtype=np.int32)
    for l in range(L):
        for u in range(S):
            kp = int(rng.integers(0, k + 1))
            topk[l, u, :kp] = rng.permutation(nb)[:kp]
    inter, total = H.overlap_counts(topk)
    io, to = O.overlap_counts(topk)
    assert np.array_equal(inter, io) and np.array_equal(total, to)
    M = H.similarity_from_counts(inter, total)
    assert M.tobytes() == O.similarity_from_counts(io, to).tobytes()
    assert M.tobytes() == H.similarity(topk).tobytes()


def test_similarity_from_counts_rejects_impossible_counts(lib):
    inter = np.array([[2, 0], [3, 2]], dtype=np.int64)
    with pytest.raises(H.HylraError):
        H.similarity_from_counts(inter, np.array([2, 2], dtype=np.int64))  # 3 > total 2
    with pytest.raises(H.HylraError):
        H.similarity_from_counts(np.array([[2, 1], [1, 2]], dtype=np.int64),
                                 np.array([2, 2], dtype=np.int64))  # above the diagonal
    M = H.similarity_from_counts(np.zeros((2, 2), dtype=np.int64), np.zeros(2, dtype=np.int64))
    assert np.all(M == 0.0)


def _dyadic(L, rng, denom=64):
    M = np.zeros((L, L))
    for t in range(L):
        M[t, :t] = rng.integers(0, denom + 1, size=t) / denom
        M[t, t] = 1.0
    return M


@pytest.mark.parametrize("L", [1, 2, 4, 7, 8])
def test_dp_matches_oracle_and_bruteforce(lib, L):
    rng = np.random.default_rng(100 + L)
    for trial in range(30):
        M = _dyadic(L, rng)
        theta = float(rng.choice([0.0, 0.3, 0.5, 0.75, 0.8, 1.0, -1.0]))
        got = H.dp_policy(M, theta)
        assert got == O.dp_policy(M, theta)
        assert got == O.dp_policy_bruteforce(M, theta)


def test_dp_matches_oracle_long(lib):
    rng = np.random.default_rng(5)
    for L in (16, 32, 64):
        M = _dyadic(L, rng, denom=16)
        for theta in (0.5, 0.8, 0.9):
            assert H.dp_policy(M, theta) == O.dp_policy(M, theta)


def test_dp_golden(lib):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "dp_4layer.json")))
    for case in g["cases"]:
        pol, R, S = H.dp_policy(np.array(g["M"]), case["theta"])
        assert list(pol) == case["policy"] and R == case["resets"] and S == case["sim"]


def test_dp_rejects_nan_theta(lib):
    with pytest.raises(H.HylraError):
        H.dp_policy(np.eye(3), float("nan"))


@pytest.mark.parametrize("L,period", [(1, 3), (4, 3), (32, 3), (32, 1), (7, 7), (5, 9)])
def test_static_policy_matches_oracle(lib, L, period):
    assert H.static_policy(L, period) == O.static_policy(L, period)


def test_static_policy_rejects_bad_period(lib):
    with pytest.raises(H.HylraError):
        H.static_policy(4, 0)


def test_jump3_against_dp_on_the_same_matrix(lib):
    """Where Jump3 is feasible under theta, the DP optimum never resets more."""
    rng = np.random.default_rng(11)
    for trial in range(40):
        L = int(rng.integers(2, 13))
        M = _dyadic(L, rng, denom=8)
        theta = float(rng.choice([0.0, 0.25, 0.5]))
        jump, Rj = H.static_policy(L, 3)
        ok, Rc, _ = O.policy_cost(M, theta, jump)
        assert Rc == Rj or not ok
        _, Rdp, _ = H.dp_policy(M, theta)
        if ok:
            assert Rdp <= Rj


def test_pooled_profiling_steps(lib):
    """Index sets of several profiled decode steps pool into one matrix: P
    copies of one step give that step's matrix; mixed steps match the oracle."""
    rng = np.random.default_rng(21)
    L, S, k, nb = 6, 8, 4, 24
    steps = []
    for p in range(3):
        t = np.empty((L, S, k), dtype=np.int32)
        for l in range(L):
            for u in range(S):
                t[l, u] = rng.permutation(nb)[:k]
        steps.append(t)
    one = H.similarity(steps[0])
    assert H.similarity(np.concatenate([steps[0]] * 3, axis=1)).tobytes() == one.tobytes()
    mixed = np.concatenate(steps, axis=1)
    assert H.similarity(mixed).tobytes() == O.similarity_matrix(mixed).tobytes()


def test_trace_build_compiles_and_exports_its_hooks(tmp_path):
    """The documented trace build (-DHYLRA_TRACE: globaltimer events, plan and
    late-start overrides) still compiles for sm_100a and exports its hooks."""
    import ctypes
    import subprocess
    from kv_cache_sparsity_b200 import build as hbuild
    out = tmp_path / "libhylra_trace.so"
    cmd = [hbuild.nvcc_path(), "-DHYLRA_TRACE", "-gencode", hbuild.GENCODE, "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", hbuild.INCLUDE, "-I", hbuild.CSRC,
           "-o", str(out)] + hbuild.SOURCES
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-3000:]
    tl = ctypes.CDLL(str(out))
    for name in ("hylra_trace_set", "hylra_plan_override", "hylra_late_override",
                 "hylra_decode_step"):
        assert hasattr(tl, name), name


@pytest.mark.parametrize("seed", range(4))
def test_token_topk_matches_oracle_ranking(lib, seed):
    """Host token selection against the oracle's ranking rule on the same
    fp32 scores (many exact ties: scores drawn from a few values)."""
    rng = np.random.default_rng(70 + seed)
    U, n, k = 6, 300, int(rng.integers(1, 40))
    scores = rng.choice(np.array([0.0, 0.125, 0.5, 0.75, 1e-7], dtype=np.float32), size=(U, n))
    scores[1] = rng.random(n).astype(np.float32)
    lengths = rng.integers(0, n + 1, size=U).astype(np.int32)
    lengths[0] = n
    got = H.token_topk(scores, k, lengths)
    for u in range(U):
        want = O.topk_blocks(scores[u, :lengths[u]], k)
        assert np.array_equal(got[u], want), u
    assert np.array_equal(H.token_topk(scores, k), np.stack([O.topk_blocks(s, k) for s in scores]))


def test_token_topk_rejects_bad_scores(lib):
    for bad in (np.nan, np.inf, -1.0):
        s = np.zeros((2, 5), dtype=np.float32)
        s[1, 3] = bad
        with pytest.raises(H.HylraError):
            H.token_topk(s, 2)
    with pytest.raises(H.HylraError):
        H.token_topk(np.zeros((1, 5), dtype=np.float32), 2, lengths=np.array([6], dtype=np.int32))


@pytest.mark.parametrize("field,limit,extra", [
    ("batch", 1024, {}), ("topk", 1024, {}),
    ("max_seqlen", 262144, {"kv_capacity": 262144 + 1}),
])
def test_limits_are_exact(lib, field, limit, extra):
    """Each documented limit is accepted and the next value rejected as
    unsupported, before anything touches a device."""
    n = ctypes.c_size_t(0)
    ok = _shape(**{field: limit, **extra})
    # accepted: past validation (without a GPU the device query then fails)
    assert lib.hylra_workspace_bytes(ctypes.byref(ok), ctypes.byref(n)) in (0, -3)
    over = _shape(**{field: limit + 1, **extra})
    assert lib.hylra_workspace_bytes(ctypes.byref(over), ctypes.byref(n)) == -2
