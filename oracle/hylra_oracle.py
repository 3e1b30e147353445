"""Plain fp64 CPU oracle for HyLRA decode attention.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import this module:
only the tests under ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library (no common helpers, headers or tables); the only
thing both sides share is the seeded input generator, which holds none of the
method's arithmetic.

Source: "HyLRA: Hybrid Layer Reuse Attention for Efficient Long-Context
Inference" (gist.science technical summary of arXiv 2602.00777), cited below
as "HyLRA summary" with its section numbers:

* §2.3 "Hybrid Inference Strategy": sensitive (reset) layers run standard
  full attention and extract top-k indices that are passed forward; tolerant
  (reuse) layers restrict attention to the subset of the KV cache named by the
  reused indices.
* §2.4 "Hardware-Efficient Optimizations", "Block-level Sparsity": the
  selection works on fixed-size token blocks of 128 tokens.
* §2.2 "Offline Policy Optimization via Dynamic Programming": the overlap
  matrix M between source and target layers and the DP over states (i, j) with
  reset jumps and vertical moves gated by a threshold theta.

Where the summary is silent the plainest reading is taken (each one is marked
READING below):

* attention scale is 1/sqrt(d); q-head g reads KV head g // r (r = Hq/Hkv);
  the decode query sees every cached token t < n (no other mask);
* a block's importance is its attention probability mass summed over the r
  q-heads sharing the KV head, computed in fp64 and rounded once to fp32;
  top-k orders by (score desc, block index asc) and pads with -1 when a
  sequence has fewer than k blocks;
* a reuse layer renormalises softmax over the selected tokens only; an empty
  selection yields a zero output;
* M[t][s] (row = target t, column = source s <= t) is the pooled overlap
  ratio sum |I_s & I_t| / sum |I_t| over the profiled index sets;
* a vertical move needs M > theta (strict); the objective is lexicographic:
  fewest resets, then largest cumulative similarity, then the
  lexicographically smallest policy string with reuse (0) before reset (1).

Parity status: every function below is pinned by tests in
``tests/test_oracle_*.py`` against closed forms, library routines (torch
``scaled_dot_product_attention`` in fp64) or exhaustive enumeration.
"""

from __future__ import annotations

import itertools
import math
from typing import Sequence

import numpy as np

BLOCK_TOKENS = 128  # HyLRA summary §2.4: fixed-size token blocks, e.g. 128 tokens

RESET = 1
REUSE = 0


# ---------------------------------------------------------------------------
# Full attention on a reset layer (HyLRA summary §2.3, "Sensitive Layers")
# ---------------------------------------------------------------------------

def attention_probs(q_g: np.ndarray, K_h: np.ndarray) -> np.ndarray:
    """Softmax probabilities of one query row over the keys ``K_h``.

    Standard scaled dot-product attention for a single decode query
    (HyLRA summary §2.3): logits l_t = q . K_t / sqrt(d), then
    p_t = exp(l_t - max l) / sum_t exp(l_t - max l).  fp64 throughout.
    """
    q_g = np.asarray(q_g, dtype=np.float64)
    K_h = np.asarray(K_h, dtype=np.float64)
    d = q_g.shape[0]
    logits = (K_h @ q_g) / math.sqrt(d)
    m = np.max(logits)
    e = np.exp(logits - m)
    return e / np.sum(e)


def full_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, n: int):
    """Full decode attention of one sequence (HyLRA summary §2.3).

    q: [Hq, d]; K, V: [Hkv, >=n, d] (only the first n tokens are the cache).
    Returns (out [Hq, d] fp64, probs [Hq, n] fp64).  q-head g uses KV head
    g // r (READING: contiguous GQA grouping).  n == 0 gives zeros.
    """
    q = np.asarray(q, dtype=np.float64)
    Hq, d = q.shape
    Hkv = K.shape[0]
    r = Hq // Hkv
    out = np.zeros((Hq, d), dtype=np.float64)
    probs = np.zeros((Hq, n), dtype=np.float64)
    if n == 0:
        return out, probs
    for g in range(Hq):
        h = g // r
        p = attention_probs(q[g], K[h, :n])
        probs[g] = p
        out[g] = p @ np.asarray(V[h, :n], dtype=np.float64)
    return out, probs


# ---------------------------------------------------------------------------
# Block scores and top-k (HyLRA summary §2.3 "top-k indices are extracted",
# §2.4 "Block-level Sparsity")
# ---------------------------------------------------------------------------

def num_blocks(n: int) -> int:
    return (n + BLOCK_TOKENS - 1) // BLOCK_TOKENS


def block_scores(probs: np.ndarray, num_kv_heads: int) -> np.ndarray:
    """fp64 attention mass of every 128-token block, per KV head.

    probs: [Hq, n] from ``full_attention``.  S[h, beta] = sum over the r
    q-heads g of KV head h and over tokens t in block beta (t < n) of
    p[g, t].  READING: the summary names block-level top-k but not the score;
    the probability mass the full layer already computes is used.
    """
    Hq, n = probs.shape
    r = Hq // num_kv_heads
    nb = num_blocks(n)
    S = np.zeros((num_kv_heads, nb), dtype=np.float64)
    for h in range(num_kv_heads):
        for beta in range(nb):
            lo = beta * BLOCK_TOKENS
            hi = min(lo + BLOCK_TOKENS, n)
            S[h, beta] = np.sum(probs[h * r:(h + 1) * r, lo:hi])
    return S


def round_scores_fp32(S: np.ndarray) -> np.ndarray:
    """Round fp64 block scores once to fp32 (round to nearest even)."""
    return np.asarray(S, dtype=np.float64).astype(np.float32)


def topk_blocks(S32: np.ndarray, k: int) -> np.ndarray:
    """Top-k block indices of one KV head, in rank order.

    Ranks blocks by fp32 score descending, equal scores by lower block index
    first (READING: tie rule not on the page).  Returns k int32 entries; the
    entries after k' = min(k, number of blocks) are -1.
    """
    nb = len(S32)
    order = sorted(range(nb), key=lambda beta: (-float(S32[beta]), beta))
    kp = min(k, nb)
    out = np.full(k, -1, dtype=np.int32)
    out[:kp] = order[:kp]
    return out


def full_layer(q, K, V, n: int, k: int):
    """Reset layer of one sequence: output, fp32 block scores and top-k.

    Returns (out [Hq, d], S32 [Hkv, NB] float32, topk [Hkv, k] int32).
    """
    Hkv = K.shape[0]
    out, probs = full_attention(q, K, V, n)
    S32 = round_scores_fp32(block_scores(probs, Hkv))
    topk = np.stack([topk_blocks(S32[h], k) for h in range(Hkv)]) if Hkv else None
    return out, S32, topk


def layer_topk(q, K, n: int, k: int):
    """The ranking half of ``full_layer``: fp32 block scores and top-k of a
    reset layer without its attention output (no V is read).  Used for
    profiling runs, where only the index sets feed the overlap matrix
    (HyLRA summary §2.2, "Similarity Matrix Construction").

    Returns (S32 [Hkv, NB] float32, topk [Hkv, k] int32), the same values as
    ``full_layer(q, K, V, n, k)[1:]``.
    """
    q = np.asarray(q, dtype=np.float64)
    Hq = q.shape[0]
    Hkv = K.shape[0]
    r = Hq // Hkv
    probs = np.zeros((Hq, n), dtype=np.float64)
    if n > 0:
        for g in range(Hq):
            probs[g] = attention_probs(q[g], K[g // r, :n])
    S32 = round_scores_fp32(block_scores(probs, Hkv))
    topk = np.stack([topk_blocks(S32[h], k) for h in range(Hkv)])
    return S32, topk


def token_scores(probs: np.ndarray, num_kv_heads: int) -> np.ndarray:
    """fp64 attention mass of every token, per KV head: S[h, t] = sum over
    the r q-heads g of KV head h of p[g, t].  The token-level counterpart of
    ``block_scores`` for a profiling run that records top-k *token* indices
    (HyLRA summary §2.2, "Similarity Matrix Construction", speaks of top-k
    token indices; the block version follows §2.4)."""
    Hq, n = probs.shape
    r = Hq // num_kv_heads
    S = np.zeros((num_kv_heads, n), dtype=np.float64)
    for h in range(num_kv_heads):
        for g in range(h * r, (h + 1) * r):
            S[h] += probs[g]
    return S


def layer_token_topk(q, K, n: int, k_tokens: int):
    """Top-k tokens of a reset layer, per KV head: fp32 token scores (fp64
    mass rounded once) ranked by score descending, lower token index first
    among equal scores, padded with -1.  Returns (S32 [Hkv, n] float32,
    topk [Hkv, k_tokens] int32)."""
    q = np.asarray(q, dtype=np.float64)
    Hq = q.shape[0]
    Hkv = K.shape[0]
    r = Hq // Hkv
    probs = np.zeros((Hq, n), dtype=np.float64)
    if n > 0:
        for g in range(Hq):
            probs[g] = attention_probs(q[g], K[g // r, :n])
    S32 = round_scores_fp32(token_scores(probs, Hkv))
    # the ranking rule is the blocks' one, applied to tokens
    topk = np.stack([topk_blocks(S32[h], k_tokens) for h in range(Hkv)])
    return S32, topk


def topk_gap(S32_h: np.ndarray, k: int) -> float:
    """Smallest relative gap between consecutive ranks 1..k'+1 of one head.

    A certificate for exact index parity: the GPU computes the same fp32
    score in another summation order, so two ranks can swap only when their
    scores are within a few ulps.  Returns +inf when there is nothing to
    separate (fewer than two candidate ranks).
    """
    s = np.sort(np.asarray(S32_h, dtype=np.float64))[::-1]
    m = min(k + 1, len(s))
    gaps = [(s[i] - s[i + 1]) / s[i] for i in range(m - 1) if s[i] > 0]
    return min(gaps) if gaps else math.inf


# ---------------------------------------------------------------------------
# Reuse layer (HyLRA summary §2.3, "Tolerant Layers")
# ---------------------------------------------------------------------------

def selected_tokens(indices: Sequence[int], n: int) -> list[int]:
    """Token positions covered by the valid block indices (-1 entries skipped)."""
    toks: list[int] = []
    for beta in indices:
        beta = int(beta)
        if beta < 0:
            continue
        lo = beta * BLOCK_TOKENS
        toks.extend(range(lo, min(lo + BLOCK_TOKENS, n)))
    return toks


def reuse_attention(q, K, V, n: int, topk: np.ndarray) -> np.ndarray:
    """Attention restricted to the reused blocks (HyLRA summary §2.3).

    topk: [Hkv, k] block indices from the most recent reset layer.  Softmax is
    taken over the selected tokens only (READING: renormalised, no extra
    sink or recent-window blocks).  An empty selection gives zeros.
    """
    q = np.asarray(q, dtype=np.float64)
    Hq, d = q.shape
    Hkv = K.shape[0]
    r = Hq // Hkv
    out = np.zeros((Hq, d), dtype=np.float64)
    for g in range(Hq):
        h = g // r
        toks = selected_tokens(topk[h], n)
        if not toks:
            continue
        p = attention_probs(q[g], np.asarray(K[h], dtype=np.float64)[toks])
        out[g] = p @ np.asarray(V[h], dtype=np.float64)[toks]
    return out


# ---------------------------------------------------------------------------
# One decode step over all layers (HyLRA summary §2.3)
# ---------------------------------------------------------------------------

def decode_step(policy: Sequence[int], layers, seqlens: Sequence[int], k: int):
    """Walk the layers under ``policy`` for a batch of sequences.

    layers[l] = (q [B, Hq, d], K [B, Hkv, >=n, d], V [B, Hkv, >=n, d]).
    A reset layer runs full attention and records its top-k; a reuse layer
    attends over the top-k recorded by the most recent reset layer (the state
    (i, j) of HyLRA summary §2.2: indices of reset layer i serve layer j).
    Returns (outs [L][B, Hq, d], topk [L][B, Hkv, k], with reuse layers'
    entries copied from the layer they reused).
    """
    L = len(policy)
    if L and policy[0] != RESET:
        raise ValueError("layer 0 must be a reset layer: no indices exist before it")
    outs, topks = [], []
    current = None
    for l in range(L):
        q, K, V = layers[l]
        B = q.shape[0]
        Hkv = K.shape[1]
        out_l = np.zeros(q.shape, dtype=np.float64)
        if policy[l] == RESET:
            current = np.full((B, Hkv, k), -1, dtype=np.int32)
            for b in range(B):
                o, _, tk = full_layer(q[b], K[b], V[b], int(seqlens[b]), k)
                out_l[b] = o
                current[b] = tk
        else:
            for b in range(B):
                out_l[b] = reuse_attention(q[b], K[b], V[b], int(seqlens[b]), current[b])
        outs.append(out_l)
        topks.append(current.copy())
    return outs, topks


# ---------------------------------------------------------------------------
# Overlap matrix (HyLRA summary §2.2, "Similarity Matrix Construction")
# ---------------------------------------------------------------------------

def similarity_matrix(topk: np.ndarray) -> np.ndarray:
    """Lower-triangular overlap matrix from profiled top-k index sets.

    topk: int array [L, S, k]: for every layer, S index sets (one per
    profiled step, sequence and KV head), -1 padded.  M[t][s] for s <= t is
    sum_u |I_s[u] & I_t[u]| / sum_u |I_t[u]| (READING: pooled overlap ratio;
    row = target layer, column = source layer).  Entries above the diagonal
    are 0; a layer with no valid index sets gets a zero row.
    """
    topk = np.asarray(topk)
    L, S = topk.shape[0], topk.shape[1]
    M = np.zeros((L, L), dtype=np.float64)
    sets = [[frozenset(int(x) for x in topk[l, u] if x >= 0) for u in range(S)]
            for l in range(L)]
    for t in range(L):
        for s in range(t + 1):
            inter = 0
            total = 0
            for u in range(S):
                inter += len(sets[s][u] & sets[t][u])
                total += len(sets[t][u])
            M[t, s] = inter / total if total else 0.0
    return M


def overlap_counts(topk: np.ndarray):
    """The two integer sums behind ``similarity_matrix``.

    topk: int array [L, S, k] as for similarity_matrix.  Returns
    (inter [L, L] int64, total [L] int64): inter[t][s] = sum_u |I_s[u] & I_t[u]|
    for s <= t (0 above the diagonal), total[t] = sum_u |I_t[u]|.  Both are
    sums over the index sets u, so the counts of disjoint groups of sets (for
    example the KV heads held by different GPUs) add up to the counts of all
    of them.
    """
    topk = np.asarray(topk)
    L, S = topk.shape[0], topk.shape[1]
    sets = [[frozenset(int(x) for x in topk[l, u] if x >= 0) for u in range(S)]
            for l in range(L)]
    inter = np.zeros((L, L), dtype=np.int64)
    total = np.zeros(L, dtype=np.int64)
    for t in range(L):
        total[t] = sum(len(sets[t][u]) for u in range(S))
        for s in range(t + 1):
            inter[t, s] = sum(len(sets[s][u] & sets[t][u]) for u in range(S))
    return inter, total


def similarity_from_counts(inter: np.ndarray, total: np.ndarray) -> np.ndarray:
    """M[t][s] = inter[t][s] / total[t] (s <= t; 0 where total[t] is 0)."""
    inter = np.asarray(inter)
    L = inter.shape[0]
    M = np.zeros((L, L), dtype=np.float64)
    for t in range(L):
        for s in range(t + 1):
            M[t, s] = int(inter[t, s]) / int(total[t]) if total[t] else 0.0
    return M


# ---------------------------------------------------------------------------
# Policy search (HyLRA summary §2.2, "Dynamic Programming")
# ---------------------------------------------------------------------------

def _better(a, b) -> bool:
    """Order of candidate paths: fewer resets, more similarity, smaller string."""
    ra, sa, pa = a
    rb, sb, pb = b
    if ra != rb:
        return ra < rb
    if sa != sb:
        return sa > sb
    return pa < pb


def dp_policy(M: np.ndarray, theta: float):
    """Optimal reset/reuse policy by dynamic programming over states (i, j).

    State (i, j): layer j uses the indices of reset layer i.  Start at (0, 0)
    (layer 0 is a reset).  From (i, j): a reset jump to (j+1, j+1) adds one
    reset; a vertical move to (i, j+1) is allowed when M[j+1][i] > theta and
    adds M[j+1][i] to the cumulative similarity.  Returns
    (policy tuple with 1 = reset / 0 = reuse, resets, cumulative similarity).
    """
    M = np.asarray(M, dtype=np.float64)
    L = M.shape[0]
    if L == 0:
        return (), 0, 0.0
    states = {0: (1, 0.0, (RESET,))}  # key: reset layer i of state (i, j)
    for j in range(L - 1):
        nxt: dict[int, tuple] = {}

        def consider(i, cand):
            if i not in nxt or _better(cand, nxt[i]):
                nxt[i] = cand

        for i, (R, S, pol) in states.items():
            consider(j + 1, (R + 1, S, pol + (RESET,)))
            if M[j + 1, i] > theta:
                consider(i, (R, S + M[j + 1, i], pol + (REUSE,)))
        states = nxt
    best = None
    for cand in states.values():
        if best is None or _better(cand, best):
            best = cand
    R, S, pol = best
    return pol, R, S


def policy_cost(M: np.ndarray, theta: float, policy: Sequence[int]):
    """(feasible, resets, cumulative similarity) of one policy string."""
    M = np.asarray(M, dtype=np.float64)
    if len(policy) == 0:
        return True, 0, 0.0
    if policy[0] != RESET:
        return False, 0, 0.0
    i = 0
    R, S = 1, 0.0
    for j in range(1, len(policy)):
        if policy[j] == RESET:
            i = j
            R += 1
        else:
            if not M[j, i] > theta:
                return False, R, S
            S += M[j, i]
    return True, R, S


def dp_policy_bruteforce(M: np.ndarray, theta: float):
    """Exhaustive search over all 2^(L-1) policies with layer 0 reset."""
    L = np.asarray(M).shape[0]
    if L == 0:
        return (), 0, 0.0
    best = None
    for tail in itertools.product((REUSE, RESET), repeat=L - 1):
        pol = (RESET,) + tail
        ok, R, S = policy_cost(M, theta, pol)
        if not ok:
            continue
        cand = (R, S, pol)
        if best is None or _better(cand, best):
            best = cand
    R, S, pol = best
    return pol, R, S


def static_policy(num_layers: int, period: int):
    """HyLRA summary §4 "Results", the Jump3 baseline ("a static variant with
    fixed jump steps"), READING: a reset every `period` layers starting at
    layer 0 (Jump3: period 3), with no similarity threshold."""
    pol = []
    for layer in range(num_layers):
        pol.append(RESET if layer % period == 0 else REUSE)
    return tuple(pol), sum(pol)
