"""Python binding of the HyLRA C-ABI library (argument marshalling only).

Every function here forwards to the entry point of the same name in
``libhylra.so`` (declared in ``include/hylra.h``).  Device buffers are torch
CUDA tensors (only their ``data_ptr()`` crosses the boundary); host buffers
for the policy functions are numpy arrays.  There is no fallback: if the
shared library is missing or a call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhylra.so")

BLOCK_TOKENS = 128
HEAD_DIM = 128
MAX_GROUP = 8
MAX_BATCH = 1024
MAX_TOPK = 1024
MAX_SEQLEN = 262144

BF16 = 0
FP32 = 1

STATUS_BAD_SEQLEN = 0x1
STATUS_BAD_INDEX = 0x2
STATUS_DUP_INDEX = 0x4
STATUS_NONFINITE = 0x8
STATUS_TIMEOUT = 0x10

ERRORS = {0: "HYLRA_OK", -1: "HYLRA_ERR_INVALID", -2: "HYLRA_ERR_UNSUPPORTED",
          -3: "HYLRA_ERR_CUDA", -4: "HYLRA_ERR_WORKSPACE"}

EXPORTS = ("hylra_workspace_bytes", "hylra_workspace_init", "hylra_decode_full",
           "hylra_decode_reuse", "hylra_decode_step", "hylra_decode_step_host",
           "hylra_similarity", "hylra_dp_policy", "hylra_read_status", "hylra_strerror",
           "hylra_version", "hylra_decode_full_noalloc", "hylra_static_policy",
           "hylra_stage_bytes", "hylra_gather_blocks", "hylra_decode_reuse_staged",
           "hylra_decode_step_offload", "hylra_overlap_counts",
           "hylra_similarity_from_counts", "hylra_set_wait_limit", "hylra_token_scores",
           "hylra_token_topk")


class HylraError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {ERRORS.get(code, code)} ({code})")
        self.code = code


class Shape(ctypes.Structure):
    """Mirror of hylra_shape_t."""

    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("max_seqlen", ctypes.c_int32),
                ("kv_capacity", ctypes.c_int64), ("total_tokens", ctypes.c_int64),
                ("seq_offsets", ctypes.c_void_p)]


def make_shape(batch, num_q_heads, num_kv_heads, topk, max_seqlen, dtype=BF16, kv_capacity=0,
               total_tokens=0, seq_offsets=None, head_dim=HEAD_DIM,
               block_size=BLOCK_TOKENS) -> Shape:
    """Build a Shape; ``seq_offsets`` is a device int64 tensor (packed layout) or None."""
    ptr = None if seq_offsets is None else int(seq_offsets.data_ptr())
    return Shape(batch, num_q_heads, num_kv_heads, head_dim, block_size, topk, dtype,
                 max_seqlen, kv_capacity, total_tokens, ptr)


_lib: Optional[ctypes.CDLL] = None


def load() -> ctypes.CDLL:
    """Load libhylra.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m kv_cache_sparsity_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, S, I32, I64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64
    SP = ctypes.POINTER(Shape)
    sig = {
        "hylra_workspace_bytes": [SP, ctypes.POINTER(ctypes.c_size_t)],
        "hylra_workspace_init": [P, S, P],
        "hylra_decode_full": [SP, P, P, P, P, P, P, P, S, P],
        "hylra_decode_reuse": [SP, P, P, P, P, P, P, P, S, P],
        "hylra_decode_step": [SP, I32, P, P, P, P, P, P, P, P, S, P],
        "hylra_decode_step_host": [SP, I32, P, P, P, P, P, P, P, P, P, P, P, S, P],
        "hylra_similarity": [I32, I32, I32, P, P],
        "hylra_overlap_counts": [I32, I32, I32, P, P, P],
        "hylra_similarity_from_counts": [I32, P, P, P],
        "hylra_dp_policy": [I32, P, ctypes.c_double, P, ctypes.POINTER(I32),
                            ctypes.POINTER(ctypes.c_double)],
        "hylra_read_status": [P, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int, P],
        "hylra_decode_full_noalloc": [SP, P, P, P, P, P, P, P, P],
        "hylra_static_policy": [I32, I32, P, ctypes.POINTER(I32)],
        "hylra_stage_bytes": [SP, ctypes.POINTER(ctypes.c_size_t)],
        "hylra_gather_blocks": [SP, P, P, P, P, P, P, P],
        "hylra_decode_reuse_staged": [SP, P, P, P, P, P, P, P, S, P],
        "hylra_decode_step_offload": [SP, I32, P, P, P, P, P, P, P, P, P, P, P, S, P],
        "hylra_set_wait_limit": [I64],
        "hylra_token_scores": [SP, P, P, P, P, P, P, P, P, S, P],
        "hylra_token_topk": [I32, I32, P, P, I32, P],
        "hylra_strerror": [ctypes.c_int],
        "hylra_version": [],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_char_p if name == "hylra_strerror" else ctypes.c_int
    _lib = lib
    return lib


def _check(rc: int, what: str):
    if rc != 0:
        raise HylraError(rc, what)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def version() -> int:
    return load().hylra_version()


def strerror(code: int) -> str:
    return load().hylra_strerror(code).decode()


def workspace_bytes(shape: Shape) -> int:
    n = ctypes.c_size_t(0)
    _check(load().hylra_workspace_bytes(ctypes.byref(shape), ctypes.byref(n)),
           "hylra_workspace_bytes")
    return n.value


def workspace_init(ws, stream=None):
    _check(load().hylra_workspace_init(_ptr(ws), ws.numel() * ws.element_size(),
                                       _stream(stream)), "hylra_workspace_init")


def decode_full(shape: Shape, q, K, V, seqlens, out, topk_out, ws, stream=None):
    _check(load().hylra_decode_full(ctypes.byref(shape), _ptr(q), _ptr(K), _ptr(V),
                                    _ptr(seqlens), _ptr(out), _ptr(topk_out), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)),
           "hylra_decode_full")


def decode_reuse(shape: Shape, q, K, V, seqlens, topk_in, out, ws, stream=None):
    _check(load().hylra_decode_reuse(ctypes.byref(shape), _ptr(q), _ptr(K), _ptr(V),
                                     _ptr(seqlens), _ptr(topk_in), _ptr(out), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)),
           "hylra_decode_reuse")


def _ptr_array(ts):
    arr = (ctypes.c_void_p * len(ts))(*[_ptr(t) for t in ts])
    return arr


def decode_step(shape: Shape, policy: Sequence[int], qs, Ks, Vs, seqlens, outs, topk, ws,
                stream=None):
    L = len(policy)
    pol = (ctypes.c_uint8 * L)(*[int(x) for x in policy])
    _check(load().hylra_decode_step(ctypes.byref(shape), L, pol, _ptr_array(qs), _ptr_array(Ks),
                                    _ptr_array(Vs), _ptr(seqlens), _ptr_array(outs), _ptr(topk),
                                    _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "hylra_decode_step")


def decode_step_host(shape: Shape, policy: Sequence[int], q_host, q_dev, Ks, Vs, seqlens,
                     out_dev, out_host, topk_dev, topk_host, ws, stream=None):
    """Step with per-step inputs/outputs in host memory (pinned torch CPU tensors)."""
    L = len(policy)
    pol = (ctypes.c_uint8 * L)(*[int(x) for x in policy])
    _check(load().hylra_decode_step_host(ctypes.byref(shape), L, pol, _ptr(q_host), _ptr(q_dev),
                                         _ptr_array(Ks), _ptr_array(Vs), _ptr(seqlens),
                                         _ptr(out_dev), _ptr(out_host), _ptr(topk_dev),
                                         _ptr(topk_host), _ptr(ws),
                                         ws.numel() * ws.element_size(), _stream(stream)),
           "hylra_decode_step_host")


def decode_full_noalloc(shape: Shape, q, K, V, seqlens, out, topk_out, status_out=None,
                        stream=None):
    """Reset layer on the library's built-in scratch (no workspace argument)."""
    _check(load().hylra_decode_full_noalloc(ctypes.byref(shape), _ptr(q), _ptr(K), _ptr(V),
                                            _ptr(seqlens), _ptr(out), _ptr(topk_out),
                                            _ptr(status_out), _stream(stream)),
           "hylra_decode_full_noalloc")


def set_wait_limit(cycles: int):
    """Limit (SM clocks) of the kernels' bounded waits for later launches;
    cycles <= 0 restores the default."""
    _check(load().hylra_set_wait_limit(int(cycles)), "hylra_set_wait_limit")


def read_status(ws, clear: bool = True, stream=None) -> int:
    v = ctypes.c_uint32(0)
    _check(load().hylra_read_status(_ptr(ws), ctypes.byref(v), int(clear), _stream(stream)),
           "hylra_read_status")
    return v.value


def token_scores(shape: Shape, q, K, V, seqlens, out, topk_out, scores, ws, stream=None):
    """Reset layer + per-token attention mass (scores: device fp32 [B][Hkv][max_seqlen])."""
    _check(load().hylra_token_scores(ctypes.byref(shape), _ptr(q), _ptr(K), _ptr(V),
                                     _ptr(seqlens), _ptr(out), _ptr(topk_out), _ptr(scores),
                                     _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "hylra_token_scores")


def token_topk(scores: np.ndarray, k: int, lengths=None) -> np.ndarray:
    """scores: fp32 [U, n] host array (lengths: int32 [U] valid entries or None)
    -> int32 [U, k] indices in rank order, -1 padded."""
    sc = np.ascontiguousarray(scores, dtype=np.float32)
    U, n = sc.shape
    ln = None if lengths is None else np.ascontiguousarray(lengths, dtype=np.int32)
    out = np.zeros((U, k), dtype=np.int32)
    _check(load().hylra_token_topk(U, n, sc.ctypes.data, None if ln is None else ln.ctypes.data,
                                   int(k), out.ctypes.data), "hylra_token_topk")
    return out


def similarity(topk: np.ndarray) -> np.ndarray:
    """topk: int32 [L, S, k] host array -> M [L, L] float64."""
    t = np.ascontiguousarray(topk, dtype=np.int32)
    L, S, k = t.shape
    M = np.zeros((L, L), dtype=np.float64)
    _check(load().hylra_similarity(L, S, k, t.ctypes.data, M.ctypes.data), "hylra_similarity")
    return M


def overlap_counts(topk: np.ndarray):
    """topk: int32 [L, S, k] host array -> (inter [L, L] int64, total [L] int64)."""
    t = np.ascontiguousarray(topk, dtype=np.int32)
    L, S, k = t.shape
    inter = np.zeros((L, L), dtype=np.int64)
    total = np.zeros(L, dtype=np.int64)
    _check(load().hylra_overlap_counts(L, S, k, t.ctypes.data, inter.ctypes.data,
                                       total.ctypes.data), "hylra_overlap_counts")
    return inter, total


def similarity_from_counts(inter: np.ndarray, total: np.ndarray) -> np.ndarray:
    """(inter [L, L], total [L]) int64 host arrays -> M [L, L] float64."""
    i = np.ascontiguousarray(inter, dtype=np.int64)
    t = np.ascontiguousarray(total, dtype=np.int64)
    L = t.shape[0]
    M = np.zeros((L, L), dtype=np.float64)
    _check(load().hylra_similarity_from_counts(L, i.ctypes.data, t.ctypes.data, M.ctypes.data),
           "hylra_similarity_from_counts")
    return M


def dp_policy(M: np.ndarray, theta: float):
    """-> (policy tuple, resets, cumulative similarity)."""
    m = np.ascontiguousarray(M, dtype=np.float64)
    L = m.shape[0]
    pol = np.zeros(L, dtype=np.uint8)
    R = ctypes.c_int32(0)
    S = ctypes.c_double(0.0)
    _check(load().hylra_dp_policy(L, m.ctypes.data, float(theta), pol.ctypes.data,
                                  ctypes.byref(R), ctypes.byref(S)), "hylra_dp_policy")
    return tuple(int(x) for x in pol), R.value, S.value


def static_policy(num_layers: int, period: int):
    """-> (policy tuple, resets): a reset every `period` layers (Jump3: 3)."""
    pol = np.zeros(num_layers, dtype=np.uint8)
    R = ctypes.c_int32(0)
    _check(load().hylra_static_policy(int(num_layers), int(period), pol.ctypes.data,
                                      ctypes.byref(R)), "hylra_static_policy")
    return tuple(int(x) for x in pol), R.value


def stage_bytes(shape: Shape) -> int:
    n = ctypes.c_size_t(0)
    _check(load().hylra_stage_bytes(ctypes.byref(shape), ctypes.byref(n)), "hylra_stage_bytes")
    return n.value


def gather_blocks(shape: Shape, K_host, V_host, seqlens, topk_in, K_stage, V_stage, stream=None):
    """K_host / V_host: pinned torch CPU tensors (the device reads them in place)."""
    _check(load().hylra_gather_blocks(ctypes.byref(shape), _ptr(K_host), _ptr(V_host),
                                      _ptr(seqlens), _ptr(topk_in), _ptr(K_stage), _ptr(V_stage),
                                      _stream(stream)), "hylra_gather_blocks")


def decode_reuse_staged(shape: Shape, q, K_stage, V_stage, seqlens, topk_in, out, ws,
                        stream=None):
    _check(load().hylra_decode_reuse_staged(ctypes.byref(shape), _ptr(q), _ptr(K_stage),
                                            _ptr(V_stage), _ptr(seqlens), _ptr(topk_in),
                                            _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                            _stream(stream)), "hylra_decode_reuse_staged")


def decode_step_offload(shape: Shape, policy: Sequence[int], qs, Ks, Vs, offloaded, seqlens,
                        outs, topk, K_stage, V_stage, ws, stream=None):
    """Ks[l] / Vs[l] of layers with offloaded[l] = 1 are pinned torch CPU tensors;
    K_stage / V_stage each hold two staging slots (2 x stage_bytes bytes)."""
    L = len(policy)
    pol = (ctypes.c_uint8 * L)(*[int(x) for x in policy])
    off = (ctypes.c_uint8 * L)(*[int(x) for x in offloaded])
    _check(load().hylra_decode_step_offload(ctypes.byref(shape), L, pol, _ptr_array(qs),
                                            _ptr_array(Ks), _ptr_array(Vs), off, _ptr(seqlens),
                                            _ptr_array(outs), _ptr(topk), _ptr(K_stage),
                                            _ptr(V_stage), _ptr(ws),
                                            ws.numel() * ws.element_size(), _stream(stream)),
           "hylra_decode_step_offload")
