"""Seeded synthetic decode workloads (inputs only, no attention arithmetic).

Both the CUDA path's tests/bench and the fp64 oracle draw their inputs from
here, so this module holds only input synthesis: random tensors with the
shapes, layouts and structure of the workloads the HyLRA summary evaluates
(long-context decoding at 8K-60K tokens, §4 "Experimental Results"), made
concrete as five named configurations.

Structure of the keys ("salient" workloads).  Per (sequence b, KV head h):
a unit direction u[b,h] shared by every layer; a salient set of 2k blocks
shared by every layer with base amplitude A ~ U[2, 6]; a per-layer drift
A_l = A + DRIFT * W_l, where W_l is a Gaussian random walk over layers (so the
top-k sets of nearby layers overlap and the overlap decays with distance;
DRIFT = 0.7 gives the 32-layer workloads about 7 reset layers at theta = 0.8).
K_l[b,h,t] = A_l[block(t)] * u[b,h] (salient blocks only) + N(0, 0.5^2);
q_l[b,g] = sqrt(d) * u[b, g // r] + N(0, 1); V_l ~ N(0, 1).

Layouts.  Dense: K, V are [B, Hkv, cap, d] (cap = max sequence length).
Packed (ragged batches): K, V are [Hkv, sum(n_b), d] with int64 row offsets
seq_offsets[b] into each KV-head plane.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

BLOCK = 128
BASE_SEED = 20260203
DRIFT = 0.7  # per-layer step of the salient amplitudes' random walk (nats)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and structure of one synthetic decode workload."""

    name: str
    batch: int
    layers: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    topk: int
    dtype: str                  # "bf16" or "fp32"
    seqlens: tuple              # per-sequence context length
    packed: bool                # packed ragged layout instead of dense
    structure: str              # "salient" or "iid"
    policy: Optional[tuple]     # fixed policy (1 = reset, 0 = reuse) or None (DP)
    theta: Optional[float]      # DP threshold when policy is None
    seed: int

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_seqlen(self) -> int:
        return max(self.seqlens) if self.seqlens else 0

    @property
    def total_tokens(self) -> int:
        return sum(self.seqlens)

    def kv_bytes_per_layer(self) -> int:
        """K+V bytes of one full layer (every cached token of every head)."""
        es = 2 if self.dtype == "bf16" else 4
        return 2 * self.num_kv_heads * self.total_tokens * self.head_dim * es

    def kv_bytes_reuse_layer(self) -> int:
        """K+V bytes a reuse layer touches (the k' selected blocks per head)."""
        es = 2 if self.dtype == "bf16" else 4
        toks = 0
        for n in self.seqlens:
            nb = (n + BLOCK - 1) // BLOCK
            kp = min(self.topk, nb)
            # selected blocks are full 128-token blocks except possibly the last
            toks += min(kp * BLOCK, n)
        return 2 * self.num_kv_heads * toks * self.head_dim * es


def _ragged_lengths(batch: int, lo: int, hi: int, seed: int) -> tuple:
    g = torch.Generator().manual_seed(seed)
    steps = (hi - lo) // BLOCK + 1
    pick = torch.randint(0, steps, (batch,), generator=g)
    return tuple(int(lo + BLOCK * int(x)) for x in pick)


def config(name: str) -> Workload:
    """The five named workloads (small parity case first)."""
    if name == "tiny":
        return Workload("tiny", 1, 4, 8, 2, 128, 8, "fp32", (4096,), False, "iid",
                        (1, 0, 0, 1), None, BASE_SEED + 0)
    if name == "llama8b_32k":
        return Workload("llama8b_32k", 1, 32, 32, 8, 128, 16, "bf16", (32768,), False,
                        "salient", None, 0.8, BASE_SEED + 1)
    if name == "llama8b_b8_64k":
        return Workload("llama8b_b8_64k", 8, 32, 32, 8, 128, 32, "bf16", (65536,) * 8,
                        False, "salient", None, 0.8, BASE_SEED + 2)
    if name == "llama8b_128k":
        return Workload("llama8b_128k", 1, 32, 32, 8, 128, 64, "bf16", (131072,), False,
                        "salient", tuple(1 if l % 4 == 0 else 0 for l in range(32)), None,
                        BASE_SEED + 3)
    if name == "ragged16":
        return Workload("ragged16", 16, 32, 32, 8, 128, 32, "bf16",
                        _ragged_lengths(16, 8192, 131072, BASE_SEED + 4), True, "salient",
                        None, 0.8, BASE_SEED + 4)
    raise KeyError(name)


CONFIG_NAMES = ("tiny", "llama8b_32k", "llama8b_b8_64k", "llama8b_128k", "ragged16")


def custom(name="custom", batch=1, layers=1, num_q_heads=8, num_kv_heads=2, head_dim=128,
           topk=4, dtype="bf16", seqlens=(1024,), packed=False, structure="salient",
           policy=None, theta=0.8, seed=1) -> Workload:
    return Workload(name, batch, layers, num_q_heads, num_kv_heads, head_dim, topk, dtype,
                    tuple(int(x) for x in seqlens), packed, structure,
                    None if policy is None else tuple(policy), theta, seed)


def scaled(w: Workload, seqlens, layers=None, name=None) -> Workload:
    """Same structure with other sequence lengths (for small parity cases)."""
    return dataclasses.replace(w, seqlens=tuple(int(x) for x in seqlens),
                               batch=len(seqlens), layers=layers or w.layers,
                               name=name or (w.name + "_scaled"))


@dataclasses.dataclass
class _Structure:
    u: torch.Tensor        # [B, Hkv, d] unit directions
    amp: torch.Tensor      # [L, B, Hkv, NBmax] per-layer block amplitude (0 = not salient)


def _structure(w: Workload) -> _Structure:
    """Layer-shared salient structure, drawn on the CPU from the workload seed."""
    g = torch.Generator().manual_seed(w.seed * 7919 + 17)
    B, H, d = w.batch, w.num_kv_heads, w.head_dim
    nbmax = max(1, (w.max_seqlen + BLOCK - 1) // BLOCK)
    u = torch.randn(B, H, d, generator=g, dtype=torch.float64)
    u = u / u.norm(dim=-1, keepdim=True)
    amp = torch.zeros(w.layers, B, H, nbmax, dtype=torch.float64)
    for b in range(B):
        nb = (w.seqlens[b] + BLOCK - 1) // BLOCK
        nsal = min(2 * w.topk, nb)
        for h in range(H):
            blocks = torch.randperm(nb, generator=g)[:nsal]
            base = 2.0 + 4.0 * torch.rand(nsal, generator=g, dtype=torch.float64)
            walk = torch.cumsum(torch.randn(w.layers, nsal, generator=g, dtype=torch.float64),
                                dim=0)
            walk[0] = 0.0
            amp[:, b, h, blocks] = base[None, :] + DRIFT * walk
    return _Structure(u.float(), amp.float())


_STRUCT_CACHE: dict = {}


def structure(w: Workload) -> _Structure:
    key = w
    if key not in _STRUCT_CACHE:
        _STRUCT_CACHE[key] = _structure(w)
    return _STRUCT_CACHE[key]


def seq_offsets(w: Workload) -> list:
    offs = [0]
    for n in w.seqlens:
        offs.append(offs[-1] + n)
    return offs


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def step_query(w: Workload, layer: int, step: int, device="cpu", heads=None):
    """The query of one layer at decode step `step` ([B][Hq][d]); step 0 is the
    query of layer_inputs.  Later steps draw fresh noise around the same
    salient directions (the cache is left as it is: over a few profiled steps
    its growth by one token each is negligible).  ``heads``: only the query
    heads of those KV heads."""
    if heads is not None:
        q = step_query(w, layer, step, device)
        return q[:, heads.start * w.group:heads.stop * w.group].contiguous()
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    B, Hq, d = w.batch, w.num_q_heads, w.head_dim
    base = (w.seed * 1000003 + layer * 101) * 4
    # step 0: the layer's own stream; later steps: a distinct 32-bit seed
    gq = _gen(device, (base + 1) ^ ((int(step) * 0x9E3779B1) & 0xFFFFFFFF))
    if w.structure == "iid":
        q = torch.randn(B, Hq, d, generator=gq, device=device)
    else:
        st = structure(w)
        u = st.u.to(device)
        q = math.sqrt(d) * u.repeat_interleave(w.group, dim=1) + torch.randn(
            B, Hq, d, generator=gq, device=device)
    return q.to(dt)


def layer_inputs(w: Workload, layer: int, device="cpu", heads=None):
    """(q, K, V) of one layer, in the workload's dtype and layout, on ``device``.

    The same (workload, layer, device type) always gives the same values.
    ``heads`` (a range of KV heads) keeps only those KV heads and their query
    heads, with the values they have in the whole layer.
    """
    if heads is not None:
        q, K, V = layer_inputs(w, layer, device)
        h0, h1 = heads.start, heads.stop
        r = w.group
        q = q[:, h0 * r:h1 * r].contiguous()
        if w.packed:
            K, V = K[h0:h1].contiguous(), V[h0:h1].contiguous()
        else:
            K, V = K[:, h0:h1].contiguous(), V[:, h0:h1].contiguous()
        return q, K, V
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    B, Hq, H, d = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim
    base = (w.seed * 1000003 + layer * 101) * 4
    gk, gv = _gen(device, base + 2), _gen(device, base + 3)
    q = step_query(w, layer, 0, device)

    def key_rows(b, n, noise):
        # noise: [H, n, d] fp32 ; add the salient part for sequence b
        if w.structure == "iid":
            return noise
        st = structure(w)
        nb = (n + BLOCK - 1) // BLOCK
        a = st.amp[layer, b, :, :nb].to(device)                  # [H, nb]
        a_tok = a.repeat_interleave(BLOCK, dim=1)[:, :n]          # [H, n]
        return 0.5 * noise + a_tok[:, :, None] * st.u[b].to(device)[:, None, :]

    if not w.packed:
        cap = w.max_seqlen
        K = torch.empty(B, H, cap, d, dtype=dt, device=device)
        V = torch.empty(B, H, cap, d, dtype=dt, device=device)
        for b in range(B):
            n = w.seqlens[b]
            nk = torch.randn(H, cap, d, generator=gk, device=device)
            nv = torch.randn(H, cap, d, generator=gv, device=device)
            K[b] = key_rows(b, cap, nk).to(dt) if n == cap else \
                torch.cat([key_rows(b, n, nk[:, :n]), nk[:, n:]], dim=1).to(dt)
            V[b] = nv.to(dt)
    else:
        tot = w.total_tokens
        K = torch.empty(H, tot, d, dtype=dt, device=device)
        V = torch.empty(H, tot, d, dtype=dt, device=device)
        offs = seq_offsets(w)
        for b in range(B):
            n = w.seqlens[b]
            nk = torch.randn(H, n, d, generator=gk, device=device)
            nv = torch.randn(H, n, d, generator=gv, device=device)
            K[:, offs[b]:offs[b] + n] = key_rows(b, n, nk).to(dt)
            V[:, offs[b]:offs[b] + n] = nv.to(dt)
    return q, K, V


def head_slice(w: Workload, K: torch.Tensor, b: int, h: int) -> torch.Tensor:
    """The first n_b cached rows [n_b, d] of sequence b, KV head h."""
    n = w.seqlens[b]
    if w.packed:
        o = seq_offsets(w)[b]
        return K[h, o:o + n]
    return K[b, h, :n]


def per_sequence(w: Workload, K: torch.Tensor, b: int) -> torch.Tensor:
    """[Hkv, n_b, d] view of sequence b in either layout."""
    n = w.seqlens[b]
    if w.packed:
        o = seq_offsets(w)[b]
        return K[:, o:o + n]
    return K[b, :, :n]
