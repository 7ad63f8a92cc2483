"""float64 CPU oracle for DuoAttention hybrid-GQA attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``duo_oracle.c`` with ctypes;
the arrays it takes are numpy arrays of raw bf16 bit patterns (``uint16``) and
it returns float64 results.  The attention definition it follows is stated in
the header of ``duo_oracle.c`` with its sources (the DuoAttention Laguna
adapter card, sections Summary and Why It Works; the Laguna sliding-window
articles; the Laguna-XS-2.1 cookbook, section 1).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "duo_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compiles duo_oracle.c into liboracle.so beside it (gcc, -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               "-o", _LIB, _SRC, "-lm"])
    return _LIB


class _Params(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("sink", ctypes.c_int32), ("recent", ctypes.c_int32),
                ("window", ctypes.c_int32), ("softmax_scale", ctypes.c_double),
                ("full_mask", ctypes.c_void_p), ("sink_logit", ctypes.c_void_p)]


class _Cache(ctypes.Structure):
    _fields_ = [("full_k", ctypes.c_void_p), ("full_v", ctypes.c_void_p),
                ("capacity", ctypes.c_int64), ("strm_k", ctypes.c_void_p),
                ("strm_v", ctypes.c_void_p), ("seq_len", ctypes.c_void_p),
                ("ring_head", ctypes.c_void_p)]


_lib = None


def _load():
    """The compiled oracle: liboracle.so, or the copy DUO_ORACLE_LIB names (the
    mutation tests point it at deliberately broken builds of duo_oracle.c)."""
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(os.environ.get("DUO_ORACLE_LIB") or build())
        P, C = ctypes.POINTER(_Params), ctypes.POINTER(_Cache)
        vp, i64 = ctypes.c_void_p, ctypes.c_int64
        lib.oracle_attended.argtypes = [P, ctypes.c_int32, i64, i64]
        lib.oracle_attended.restype = ctypes.c_int
        lib.oracle_count_pairs.argtypes = [P, ctypes.c_int32, i64]
        lib.oracle_count_pairs.restype = i64
        lib.oracle_head_kind.argtypes = [P, ctypes.c_int32]
        lib.oracle_head_kind.restype = ctypes.c_int
        lib.oracle_attn_prefill.argtypes = [P, vp, vp, vp, i64, vp, i64, vp, vp]
        lib.oracle_attn_prefill.restype = ctypes.c_int
        lib.oracle_kv_append.argtypes = [P, C, vp, vp, ctypes.c_int32]
        lib.oracle_kv_append.restype = ctypes.c_int
        lib.oracle_attn_decode.argtypes = [P, C, vp, vp, i64, vp, vp]
        lib.oracle_attn_decode.restype = ctypes.c_int
        lib.oracle_attn_decode_block.argtypes = [P, C, vp, vp, vp, ctypes.c_int32, vp, i64, vp, vp]
        lib.oracle_attn_decode_block.restype = ctypes.c_int
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


@dataclass
class Layer:
    """One attention layer as the oracle sees it.

    window > 0 makes a sliding-window layer (every KV head keeps the last
    `window` tokens); window == 0 makes a DuoAttention layer whose KV heads
    are full-context where ``full_mask`` is 1 and streaming (sink + recent)
    elsewhere.  ``sink_logit`` (one float per query head) joins the softmax
    denominator with a zero value when given.
    """
    batch: int
    num_q_heads: int = 48
    num_kv_heads: int = 8
    head_dim: int = 128
    sink: int = 64
    recent: int = 256
    window: int = 0
    softmax_scale: float = 128 ** -0.5
    full_mask: Sequence[int] = (0,) * 8
    sink_logit: Optional[np.ndarray] = None

    def _c(self):
        mask = np.ascontiguousarray(np.asarray(self.full_mask, dtype=np.uint8))
        sl = None if self.sink_logit is None else np.ascontiguousarray(
            np.asarray(self.sink_logit, dtype=np.float32))
        keep = (mask, sl)
        p = _Params(self.batch, self.num_q_heads, self.num_kv_heads, self.head_dim,
                    self.sink, self.recent, self.window, float(self.softmax_scale),
                    mask.ctypes.data, None if sl is None else sl.ctypes.data)
        return p, keep

    @property
    def n_full(self) -> int:
        return 0 if self.window > 0 else int(sum(1 for m in self.full_mask if m))

    @property
    def n_ring(self) -> int:
        return self.num_kv_heads - self.n_full

    @property
    def ring_slots(self) -> int:
        return self.window if self.window > 0 else self.sink + self.recent


def _u16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs are passed as uint16 bit patterns")
    return a


def attended(layer: Layer, kv_head: int, i: int, j: int) -> bool:
    p, keep = layer._c()
    return bool(_load().oracle_attended(ctypes.byref(p), kv_head, i, j))


def count_pairs(layer: Layer, kv_head: int, L: int) -> int:
    p, keep = layer._c()
    return int(_load().oracle_count_pairs(ctypes.byref(p), kv_head, L))


def head_kind(layer: Layer, kv_head: int) -> int:
    """0 = full-context, 1 = streaming, 2 = sliding window."""
    p, keep = layer._c()
    return int(_load().oracle_head_kind(ctypes.byref(p), kv_head))


def attn_prefill(layer: Layer, q, k, v, rows=None):
    """Prefill attention.  q: [B][L][Hq][D], k/v: [B][L][Hkv][D] uint16 bits.

    rows: optional flat row ids (b*Hq + h)*L + i.  Returns (out [n][D], lse [n])
    in float64, rows in the order given (all rows in (b, h, i) order if None).
    """
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, L, Hq, D = q.shape
    n = B * Hq * L if rows is None else len(rows)
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    p, keep = layer._c()
    rc = _load().oracle_attn_prefill(ctypes.byref(p), q.ctypes.data, k.ctypes.data,
                                     v.ctypes.data, L, None if r is None else r.ctypes.data,
                                     n, out.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_attn_prefill failed ({rc})")
    return out, lse


class Cache:
    """Host KV cache in the head-major layout (numpy, bf16 bits)."""

    def __init__(self, layer: Layer, capacity: int):
        B, D = layer.batch, layer.head_dim
        self.capacity = capacity
        self.full_k = np.zeros((B, layer.n_full, capacity, D), dtype=np.uint16)
        self.full_v = np.zeros_like(self.full_k)
        self.strm_k = np.zeros((B, layer.n_ring, layer.ring_slots, D), dtype=np.uint16)
        self.strm_v = np.zeros_like(self.strm_k)
        self.seq_len = np.zeros((B,), dtype=np.int32)
        self.ring_head = np.zeros((B,), dtype=np.int32)

    def _c(self):
        for name in ("full_k", "full_v", "strm_k", "strm_v", "seq_len", "ring_head"):
            setattr(self, name, np.ascontiguousarray(getattr(self, name)))
        return _Cache(self.full_k.ctypes.data, self.full_v.ctypes.data, self.capacity,
                      self.strm_k.ctypes.data, self.strm_v.ctypes.data,
                      self.seq_len.ctypes.data, self.ring_head.ctypes.data)


def kv_append(layer: Layer, cache: Cache, k, v) -> None:
    """Sequential append of k/v [B][n_new][Hkv][D] (uint16 bits) into cache."""
    k, v = _u16(k), _u16(v)
    p, keep = layer._c()
    c = cache._c()
    rc = _load().oracle_kv_append(ctypes.byref(p), ctypes.byref(c), k.ctypes.data,
                                  v.ctypes.data, int(k.shape[1]))
    if rc != 0:
        raise ValueError(f"oracle_kv_append failed ({rc}): capacity exceeded")


def attn_decode(layer: Layer, cache: Cache, q, rows=None):
    """One-token decode.  q: [B][Hq][D] uint16 bits; rows: flat ids b*Hq + h."""
    q = _u16(q)
    B, Hq, D = q.shape
    n = B * Hq if rows is None else len(rows)
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    p, keep = layer._c()
    c = cache._c()
    rc = _load().oracle_attn_decode(ctypes.byref(p), ctypes.byref(c), q.ctypes.data,
                                    None if r is None else r.ctypes.data, n,
                                    out.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_attn_decode failed ({rc})")
    return out, lse


def attn_decode_block(layer: Layer, cache: Cache, q, kb, vb, rows=None):
    """Block (verify) decode against the cache before the block is appended.
    q: [B][k][Hq][D], kb/vb: [B][k][Hkv][D] uint16 bits; query t of sequence b
    is at position seq_len[b] + t.  rows: flat ids (b*k + t)*Hq + h.  Returns
    (out [n][D], lse [n]) in float64."""
    q, kb, vb = _u16(q), _u16(kb), _u16(vb)
    B, k, Hq, D = q.shape
    n = B * k * Hq if rows is None else len(rows)
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    p, keep = layer._c()
    c = cache._c()
    rc = _load().oracle_attn_decode_block(ctypes.byref(p), ctypes.byref(c), q.ctypes.data,
                                          kb.ctypes.data, vb.ctypes.data, int(k),
                                          None if r is None else r.ctypes.data, n,
                                          out.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_attn_decode_block failed ({rc})")
    return out, lse


# ------------------------------------------------------------------ output gate
# Laguna's optional attention output gate (the Laguna attention article
# "深入理解Laguna的注意力机制", section on attention output gating: one gate per
# (head, channel) or one per head broadcast over the channels; the Laguna XS
# 2.1 sliding-window article: the g_proj gate on the attention output).  The
# pages do not name the activation; the reading taken is the logistic sigmoid,
# applied to the normalised attention output: out * 1 / (1 + exp(-g)).

GATE_NONE, GATE_PER_ELEMENT, GATE_PER_HEAD = 0, 1, 2


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sigmoid(x: np.ndarray) -> np.ndarray:
    """The logistic function in float64 (exp overflow for very negative x gives 0)."""
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def gate_prefill(out: np.ndarray, gate, mode: int, L: int, Hq: int, rows=None) -> np.ndarray:
    """Gated prefill output.  out: [n][D] float64 rows as attn_prefill returns
    them (ids (b*Hq + h)*L + i); gate: bf16 bits [B][L][Hq][D] (per element) or
    [B][L][Hq] (per head)."""
    if mode == GATE_NONE:
        return out
    g = bf16_bits_to_f64(gate)
    r = np.arange(out.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    i, h, b = r % L, (r // L) % Hq, r // (L * Hq)
    gv = g[b, i, h, :] if mode == GATE_PER_ELEMENT else g[b, i, h][:, None]
    return out * sigmoid(gv)


def gate_decode(out: np.ndarray, gate, mode: int, Hq: int, rows=None) -> np.ndarray:
    """Gated decode output.  out: [n][D] rows with ids b*Hq + h; gate: bf16 bits
    [B][Hq][D] (per element) or [B][Hq] (per head)."""
    if mode == GATE_NONE:
        return out
    g = bf16_bits_to_f64(gate)
    r = np.arange(out.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    h, b = r % Hq, r // Hq
    gv = g[b, h, :] if mode == GATE_PER_ELEMENT else g[b, h][:, None]
    return out * sigmoid(gv)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))
