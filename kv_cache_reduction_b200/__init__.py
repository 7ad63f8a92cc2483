"""B200-native (sm_100a) DuoAttention hybrid-GQA attention.

Thin ctypes binding over ``libduoattn.so`` (the C ABI declared in
``include/duo_attn.h``).  The functions below carry the C names and only
marshal arguments: torch tensors are passed as device pointers and the
current CUDA stream as the stream handle.  Every step of the attention runs
in the library's CUDA kernels; there is no Python or CPU fallback, and a
missing library raises ``DuoLibraryMissing``.  Before a call reaches the
library, the binding checks what plain pointers cannot carry: each tensor's
dtype, shape, contiguity and device (the current CUDA device), raising
``ValueError``; the library checks the rest and raises ``DuoError``.

Layouts (bf16 unless noted):
  prefill  q [B][L][Hq][D], k/v [B][L][Hkv][D] -> out [B][L][Hq][D], lse fp32 [B][Hq][L]
  append   k/v [B][n_new][Hkv][D] into the cache
  decode   q [B][Hq][D] -> out [B][Hq][D], lse fp32 [B][Hq]
  cache    full_k/v [B][n_full][capacity][D], strm_k/v [B][n_ring][ring_slots][D],
           seq_len, ring_head int32 [B]
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_HERE, "libduoattn.so")

DUO_OK = 0
DUO_ERR_INVALID_ARG = -1
DUO_ERR_UNSUPPORTED = -2
DUO_ERR_CUDA = -3
DUO_ERR_WORKSPACE = -4
DUO_ERR_TIMEOUT = -5
DUO_ERR_CAPACITY = -6
DUO_ERR_DEVICE = -7

EXPORTED = ("duo_kv_append", "duo_kv_append_prep", "duo_prefill_workspace_bytes", "duo_attn_prefill",
            "duo_decode_workspace_bytes", "duo_attn_decode", "duo_decode_block_workspace_bytes",
            "duo_attn_decode_block",
            "duo_attn_decode_static", "duo_cache_bytes", "duo_get_device_status",
            "duo_status_string", "duo_last_error", "duo_testing_withhold_tile", "duo_testing_ex2")

# kernels the failure-injection hook (include/duo_attn_testing.h) can select
DUO_TESTING_DECODE, DUO_TESTING_PREFILL, DUO_TESTING_DECODE_BLOCK = 1, 2, 3


class DuoLibraryMissing(RuntimeError):
    pass


class DuoError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"{message} (code {code})")
        self.code = code


DUO_GATE_NONE, DUO_GATE_PER_ELEMENT, DUO_GATE_PER_HEAD = 0, 1, 2


class _Gate(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("values", ctypes.c_void_p)]


def _gate(gate: Optional[torch.Tensor], out: torch.Tensor):
    """A duo_gate for gate pre-activations shaped like out (one per channel) or
    like out without its last dimension (one per head); None for no gate."""
    if gate is None:
        return None
    if tuple(gate.shape) == tuple(out.shape):
        mode = DUO_GATE_PER_ELEMENT
    elif tuple(gate.shape) == tuple(out.shape[:-1]):
        mode = DUO_GATE_PER_HEAD
    else:
        raise ValueError(f"gate shape {tuple(gate.shape)} is neither out's {tuple(out.shape)} "
                         f"nor out's without the channel dimension")
    if gate.dtype != torch.bfloat16 or not gate.is_contiguous():
        raise ValueError("gate must be a contiguous bf16 tensor")
    return ctypes.byref(_Gate(mode, _ptr(gate)))


class _Prep(ctypes.Structure):
    _fields_ = [("rope_theta", ctypes.c_float), ("rope_factor", ctypes.c_float),
                ("original_max_position", ctypes.c_int32), ("beta_fast", ctypes.c_float),
                ("beta_slow", ctypes.c_float), ("attention_factor", ctypes.c_float),
                ("rms_eps", ctypes.c_float), ("q_norm_weight", ctypes.c_void_p),
                ("k_norm_weight", ctypes.c_void_p)]


@dataclass
class DuoQKPrep:
    """RMSNorm + YaRN RoPE of the new queries and keys (duo_qk_prep).  The
    defaults are the full-attention layers' rope parameters printed on the
    Laguna attention page; eps 1e-6 is a reading.  Norm weights: device bf16
    [128] tensors or None (unit weight)."""
    rope_theta: float = 500000.0
    rope_factor: float = 64.0
    original_max_position: int = 4096
    beta_fast: float = 64.0
    beta_slow: float = 1.0
    attention_factor: float = 1.0
    rms_eps: float = 1e-6
    q_norm_weight: Optional[torch.Tensor] = None
    k_norm_weight: Optional[torch.Tensor] = None

    def as_c(self) -> _Prep:
        return _Prep(self.rope_theta, self.rope_factor, self.original_max_position, self.beta_fast,
                     self.beta_slow, self.attention_factor, self.rms_eps,
                     _arg(self.q_norm_weight, "q_norm_weight", torch.bfloat16, (128,), optional=True),
                     _arg(self.k_norm_weight, "k_norm_weight", torch.bfloat16, (128,), optional=True))


class _Params(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("sink", ctypes.c_int32), ("recent", ctypes.c_int32),
                ("window", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("full_mask", ctypes.c_void_p), ("sink_logit", ctypes.c_void_p)]


class CacheStats(ctypes.Structure):
    _fields_ = [("duo_bytes", ctypes.c_uint64), ("full_cache_bytes", ctypes.c_uint64),
                ("active_bytes", ctypes.c_uint64), ("utilization", ctypes.c_double)]


class _Cache(ctypes.Structure):
    _fields_ = [("full_k", ctypes.c_void_p), ("full_v", ctypes.c_void_p),
                ("capacity", ctypes.c_int64), ("strm_k", ctypes.c_void_p),
                ("strm_v", ctypes.c_void_p), ("seq_len", ctypes.c_void_p),
                ("ring_head", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIBRARY_PATH) -> ctypes.CDLL:
    """Loads libduoattn.so (raises DuoLibraryMissing if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise DuoLibraryMissing(
            f"{path} is missing: build it with `python -m kv_cache_reduction_b200.build`")
    lib = ctypes.CDLL(path)
    P, C, vp = ctypes.POINTER(_Params), ctypes.POINTER(_Cache), ctypes.c_void_p
    lib.duo_kv_append.argtypes = [P, C, vp, vp, ctypes.c_int32, vp]
    lib.duo_kv_append.restype = ctypes.c_int
    lib.duo_kv_append_prep.argtypes = [P, C, ctypes.POINTER(_Prep), vp, vp, vp, ctypes.c_int32, vp]
    lib.duo_kv_append_prep.restype = ctypes.c_int
    lib.duo_prefill_workspace_bytes.argtypes = []
    lib.duo_prefill_workspace_bytes.restype = ctypes.c_size_t
    G = ctypes.POINTER(_Gate)
    lib.duo_attn_prefill.argtypes = [P, vp, vp, vp, ctypes.c_int32, vp, vp, vp, ctypes.c_size_t, G, vp]
    lib.duo_attn_prefill.restype = ctypes.c_int
    lib.duo_decode_workspace_bytes.argtypes = [P, ctypes.c_int32]
    lib.duo_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.duo_attn_decode.argtypes = [P, C, vp, ctypes.c_int32, vp, vp, vp, ctypes.c_size_t, G, vp]
    lib.duo_attn_decode.restype = ctypes.c_int
    lib.duo_attn_decode_static.argtypes = [P, C, vp, ctypes.c_int32, vp, vp, G, vp]
    lib.duo_decode_block_workspace_bytes.argtypes = [P, ctypes.c_int32, ctypes.c_int32]
    lib.duo_decode_block_workspace_bytes.restype = ctypes.c_size_t
    lib.duo_attn_decode_block.argtypes = [P, C, vp, vp, vp, ctypes.c_int32, ctypes.c_int32, vp, vp, vp,
                                          ctypes.c_size_t, G, vp]
    lib.duo_attn_decode_block.restype = ctypes.c_int
    lib.duo_attn_decode_static.restype = ctypes.c_int
    lib.duo_cache_bytes.argtypes = [P, ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(CacheStats)]
    lib.duo_cache_bytes.restype = ctypes.c_int
    lib.duo_get_device_status.argtypes = [vp]
    lib.duo_get_device_status.restype = ctypes.c_int
    lib.duo_status_string.argtypes = [ctypes.c_int]
    lib.duo_status_string.restype = ctypes.c_char_p
    lib.duo_last_error.argtypes = []
    lib.duo_last_error.restype = ctypes.c_char_p
    lib.duo_testing_withhold_tile.argtypes = [ctypes.c_int32, ctypes.c_int32]
    lib.duo_testing_withhold_tile.restype = ctypes.c_int
    lib.duo_testing_ex2.argtypes = [vp, vp, ctypes.c_int64, vp]
    lib.duo_testing_ex2.restype = ctypes.c_int
    _lib = lib
    return lib


@dataclass
class DuoParams:
    """One attention layer (mirrors ``duo_params``).

    ``full_mask`` is a host sequence of 0/1 per KV head (ignored when
    window > 0); ``sink_logit`` is a device fp32 tensor [Hq] or None.
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
    sink_logit: Optional[torch.Tensor] = None
    _mask_buf: ctypes.Array = field(default=None, repr=False, compare=False)

    def as_c(self) -> _Params:
        self._mask_buf = (ctypes.c_uint8 * max(1, len(self.full_mask)))(*[int(m) for m in self.full_mask])
        return _Params(self.batch, self.num_q_heads, self.num_kv_heads, self.head_dim, self.sink,
                       self.recent, self.window, float(self.softmax_scale),
                       ctypes.addressof(self._mask_buf),
                       _arg(self.sink_logit, "sink_logit", torch.float32, (self.num_q_heads,),
                            optional=True))

    @property
    def n_full(self) -> int:
        return 0 if self.window > 0 else sum(1 for m in self.full_mask if m)

    @property
    def n_ring(self) -> int:
        return self.num_kv_heads - self.n_full

    @property
    def ring_slots(self) -> int:
        return self.window if self.window > 0 else self.sink + self.recent


@dataclass
class DuoCache:
    """Device KV cache of one layer (mirrors ``duo_cache``); tensors are caller-owned."""
    full_k: Optional[torch.Tensor]
    full_v: Optional[torch.Tensor]
    capacity: int
    strm_k: Optional[torch.Tensor]
    strm_v: Optional[torch.Tensor]
    seq_len: torch.Tensor
    ring_head: torch.Tensor

    @staticmethod
    def allocate(params: DuoParams, capacity: int, device="cuda") -> "DuoCache":
        B, D = params.batch, params.head_dim
        kw = dict(dtype=torch.bfloat16, device=device)
        fk = torch.empty((B, params.n_full, capacity, D), **kw) if params.n_full else None
        fv = torch.empty_like(fk) if fk is not None else None
        sk = torch.empty((B, params.n_ring, params.ring_slots, D), **kw) if params.n_ring else None
        sv = torch.empty_like(sk) if sk is not None else None
        return DuoCache(fk, fv, capacity, sk, sv,
                        torch.zeros((B,), dtype=torch.int32, device=device),
                        torch.zeros((B,), dtype=torch.int32, device=device))

    def as_c(self, params: Optional["DuoParams"] = None) -> _Cache:
        """The duo_cache; with params, each tensor is checked against the layer's
        geometry first (a part the layer does not use is passed as NULL)."""
        if params is None:
            return _Cache(_ptr(self.full_k), _ptr(self.full_v), int(self.capacity), _ptr(self.strm_k),
                          _ptr(self.strm_v), _ptr(self.seq_len), _ptr(self.ring_head))
        B, D, bf = params.batch, params.head_dim, torch.bfloat16
        full = (B, params.n_full, int(self.capacity), D)
        ring = (B, params.n_ring, params.ring_slots, D)
        fk = _arg(self.full_k, "cache.full_k", bf, full) if params.n_full else None
        fv = _arg(self.full_v, "cache.full_v", bf, full) if params.n_full else None
        sk = _arg(self.strm_k, "cache.strm_k", bf, ring) if params.n_ring else None
        sv = _arg(self.strm_v, "cache.strm_v", bf, ring) if params.n_ring else None
        return _Cache(fk, fv, int(self.capacity), sk, sv,
                      _arg(self.seq_len, "cache.seq_len", torch.int32, (B,)),
                      _arg(self.ring_head, "cache.ring_head", torch.int32, (B,)))


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _on_device(t: torch.Tensor, name: str) -> None:
    """A tensor the kernels will read or write: contiguous and on the current
    CUDA device (a host or another GPU's pointer would fault in the kernel)."""
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    cur = torch.cuda.current_device()
    if t.device.index is not None and t.device.index != cur:
        raise ValueError(f"{name} is on {t.device}, but the current CUDA device is cuda:{cur}")


def _arg(t: Optional[torch.Tensor], name: str, dtype: torch.dtype, shape, optional: bool = False):
    """The device pointer of t after checking its dtype, its shape (None leaves
    a dimension free), contiguity and device; None for an optional None."""
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} (got {t.dtype})")
    if t.dim() != len(shape) or any(s is not None and int(d) != s for d, s in zip(t.shape, shape)):
        want = "[" + ", ".join("*" if s is None else str(s) for s in shape) + "]"
        raise ValueError(f"{name} has shape {list(t.shape)}, expected {want}")
    _on_device(t, name)
    return t.data_ptr()


def _workspace(ws: Optional[torch.Tensor]):
    """(pointer, bytes) of a workspace tensor (any dtype), or (None, 0)."""
    if ws is None:
        return None, 0
    _on_device(ws, "workspace")
    return ws.data_ptr(), ws.numel() * ws.element_size()


def _one_token(params: "DuoParams", t: Optional[torch.Tensor], name: str, dtype: torch.dtype,
               tail, optional: bool = False):
    """A one-token decode tensor: [B][tail...] or [B][1][tail...]."""
    lead = (params.batch, 1) if t is not None and t.dim() == 2 + len(tail) else (params.batch,)
    return _arg(t, name, dtype, lead + tuple(tail), optional)


def _gate_arg(gate: Optional[torch.Tensor], out: torch.Tensor):
    if gate is not None:
        _on_device(gate, "gate")
    return _gate(gate, out)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(rc: int) -> int:
    if rc < 0:
        lib = load_library()
        raise DuoError(rc, (lib.duo_last_error() or b"").decode() or
                       lib.duo_status_string(rc).decode())
    return rc


def duo_kv_append(params: DuoParams, cache: DuoCache, k: torch.Tensor, v: torch.Tensor,
                  n_new: Optional[int] = None, stream=None) -> None:
    n_new = int(k.shape[1]) if n_new is None else int(n_new)
    p, c = params.as_c(), cache.as_c(params)
    shape = (params.batch, n_new, params.num_kv_heads, params.head_dim)
    _check(load_library().duo_kv_append(ctypes.byref(p), ctypes.byref(c),
                                        _arg(k, "k", torch.bfloat16, shape),
                                        _arg(v, "v", torch.bfloat16, shape), n_new, _stream(stream)))


def duo_kv_append_prep(params: DuoParams, cache: DuoCache, prep: DuoQKPrep, q: torch.Tensor,
                       k: torch.Tensor, v: torch.Tensor, n_new: Optional[int] = None,
                       stream=None) -> None:
    """RMSNorm + YaRN RoPE of q [B][n][Hq][D] and k [B][n][Hkv][D] in place at
    positions seq_len[b] + t, then the append of the prepared k with v."""
    n_new = int(k.shape[1]) if n_new is None else int(n_new)
    p, c, pr = params.as_c(), cache.as_c(params), prep.as_c()
    B, D, bf = params.batch, params.head_dim, torch.bfloat16
    kv = (B, n_new, params.num_kv_heads, D)
    _check(load_library().duo_kv_append_prep(ctypes.byref(p), ctypes.byref(c), ctypes.byref(pr),
                                             _arg(q, "q", bf, (B, n_new, params.num_q_heads, D)),
                                             _arg(k, "k", bf, kv), _arg(v, "v", bf, kv), n_new,
                                             _stream(stream)))


def duo_prefill_workspace_bytes() -> int:
    return int(load_library().duo_prefill_workspace_bytes())


def duo_attn_prefill(params: DuoParams, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                     out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                     seq_len: Optional[int] = None, stream=None,
                     workspace: Optional[torch.Tensor] = None,
                     gate: Optional[torch.Tensor] = None) -> None:
    """workspace: None (static work-tile order) or a device tensor of at least
    duo_prefill_workspace_bytes() bytes (dynamic, balanced order).  gate: None,
    or bf16 gate pre-activations [B][L][Hq][D] (per channel) or [B][L][Hq] (per
    head); out is then multiplied by sigmoid(gate)."""
    Lq = int(q.shape[1]) if q is not None and q.dim() == 4 else -1
    L = Lq if seq_len is None else int(seq_len)
    if L not in (0, Lq):
        raise ValueError(f"seq_len {L} must be q's length {Lq} (or 0 for an empty prompt)")
    p = params.as_c()
    B, D, bf = params.batch, params.head_dim, torch.bfloat16
    qs, kvs = (B, Lq, params.num_q_heads, D), (B, Lq, params.num_kv_heads, D)
    ws, nbytes = _workspace(workspace)
    _check(load_library().duo_attn_prefill(ctypes.byref(p), _arg(q, "q", bf, qs), _arg(k, "k", bf, kvs),
                                           _arg(v, "v", bf, kvs), L, _arg(out, "out", bf, qs),
                                           _arg(lse, "lse", torch.float32, (B, params.num_q_heads, Lq),
                                                optional=True),
                                           ws, nbytes, _gate_arg(gate, out), _stream(stream)))


def duo_decode_workspace_bytes(params: DuoParams, max_seq_len: int) -> int:
    p = params.as_c()
    return int(load_library().duo_decode_workspace_bytes(ctypes.byref(p), int(max_seq_len)))


def duo_attn_decode(params: DuoParams, cache: DuoCache, q: torch.Tensor, max_seq_len: int,
                    out: torch.Tensor, lse: Optional[torch.Tensor], workspace: torch.Tensor,
                    stream=None, gate: Optional[torch.Tensor] = None) -> None:
    """gate: None, or bf16 gate pre-activations [B][Hq][D] or [B][Hq]."""
    p, c = params.as_c(), cache.as_c(params)
    Hq, D, bf = params.num_q_heads, params.head_dim, torch.bfloat16
    ws, nbytes = _workspace(workspace)
    _check(load_library().duo_attn_decode(ctypes.byref(p), ctypes.byref(c), _one_token(params, q, "q", bf, (Hq, D)),
                                          int(max_seq_len), _one_token(params, out, "out", bf, (Hq, D)),
                                          _one_token(params, lse, "lse", torch.float32, (Hq,), optional=True),
                                          ws, nbytes, _gate_arg(gate, out), _stream(stream)))


def duo_decode_block_workspace_bytes(params: DuoParams, q_len: int, max_seq_len: int) -> int:
    p = params.as_c()
    return int(load_library().duo_decode_block_workspace_bytes(ctypes.byref(p), int(q_len),
                                                               int(max_seq_len)))


def duo_attn_decode_block(params: DuoParams, cache: DuoCache, q: torch.Tensor, k_new: torch.Tensor,
                          v_new: torch.Tensor, max_seq_len: int, out: torch.Tensor,
                          lse: Optional[torch.Tensor], workspace: torch.Tensor, stream=None,
                          gate: Optional[torch.Tensor] = None) -> None:
    """Block decode: q [B][k][Hq][D] at positions seq_len[b] + t against the
    cache plus the block's own k_new / v_new [B][k][Hkv][D]; the cache is not
    modified.  k <= 8 is a verify block; longer blocks (chunked prefill: a
    prompt chunk continuing cached tokens) take the two-pass prefill path."""
    p, c = params.as_c(), cache.as_c(params)
    B, D, bf = params.batch, params.head_dim, torch.bfloat16
    k = int(q.shape[1]) if q is not None and q.dim() == 4 else -1
    qs, kvs = (B, k, params.num_q_heads, D), (B, k, params.num_kv_heads, D)
    ws, nbytes = _workspace(workspace)
    _check(load_library().duo_attn_decode_block(ctypes.byref(p), ctypes.byref(c), _arg(q, "q", bf, qs),
                                                _arg(k_new, "k_new", bf, kvs), _arg(v_new, "v_new", bf, kvs),
                                                k, int(max_seq_len), _arg(out, "out", bf, qs),
                                                _arg(lse, "lse", torch.float32, (B, k, params.num_q_heads),
                                                     optional=True),
                                                ws, nbytes, _gate_arg(gate, out), _stream(stream)))


def duo_attn_decode_static(params: DuoParams, cache: DuoCache, q: torch.Tensor, max_seq_len: int,
                           out: torch.Tensor, lse: Optional[torch.Tensor], stream=None,
                           gate: Optional[torch.Tensor] = None) -> None:
    """duo_attn_decode with the library's built-in 16 MiB scratch instead of a
    caller workspace, for callers that cannot allocate device memory when they
    decode.  Calls that may overlap on the GPU share that scratch and race."""
    p, c = params.as_c(), cache.as_c(params)
    Hq, D, bf = params.num_q_heads, params.head_dim, torch.bfloat16
    _check(load_library().duo_attn_decode_static(
        ctypes.byref(p), ctypes.byref(c), _one_token(params, q, "q", bf, (Hq, D)), int(max_seq_len),
        _one_token(params, out, "out", bf, (Hq, D)),
        _one_token(params, lse, "lse", torch.float32, (Hq,), optional=True),
        _gate_arg(gate, out), _stream(stream)))


def duo_cache_bytes(params: DuoParams, capacity: int, seq_len: int) -> CacheStats:
    """KV-cache size of a layer against a full cache, and its active utilisation
    when every sequence holds seq_len tokens (host arithmetic)."""
    p, st = params.as_c(), CacheStats()
    _check(load_library().duo_cache_bytes(ctypes.byref(p), int(capacity), int(seq_len),
                                          ctypes.byref(st)))
    return st


def duo_get_device_status(stream=None) -> int:
    return int(load_library().duo_get_device_status(_stream(stream)))


def duo_status_string(code: int) -> str:
    return load_library().duo_status_string(int(code)).decode()


def duo_last_error() -> str:
    return (load_library().duo_last_error() or b"").decode()


def duo_testing_withhold_tile(kernel: int, tile: int) -> None:
    """Failure injection for tests (include/duo_attn_testing.h): CTA 0's tile
    producer of the selected kernel stops before its tile-th tile, so the
    kernel's bounded waits expire and the call's status reads DUO_ERR_TIMEOUT.
    tile = -1 turns it off."""
    _check(load_library().duo_testing_withhold_tile(int(kernel), int(tile)))


def duo_testing_ex2(x: torch.Tensor, stream=None) -> torch.Tensor:
    """2^x by the prefill's FMA-pipe exponential (include/duo_attn_testing.h),
    for tests of its error bound: x a contiguous fp32 CUDA tensor."""
    if x.dtype != torch.float32:
        raise ValueError("x must be float32")
    _on_device(x, "x")
    y = torch.empty_like(x)
    _check(load_library().duo_testing_ex2(x.data_ptr(), y.data_ptr(), x.numel(), _stream(stream)))
    return y


def workspace_for(params: DuoParams, max_seq_len: int, device="cuda") -> torch.Tensor:
    """Allocates a zero-filled decode workspace of the size the library asks for
    (torch memory).  It may be reused by any later call that fits in it."""
    n = max(duo_decode_workspace_bytes(params, max_seq_len), 256)
    return torch.zeros((n + 255) // 256 * 256, dtype=torch.uint8, device=device)
