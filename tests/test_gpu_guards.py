"""Out-of-bounds write checks: every output, cache, in-place input and
workspace of the kernels sits between guard regions (tests/guards.py), and
after each call the guards must be untouched.  The cases are the ones where an
index error would show first: ragged prefills, bulk appends longer than the
ring, an append that stops at the capacity, the fused prep with the ring
wrapping, the verify block at its widest, and decodes with empty sequences.
Each call's result is also compared with the oracle, so the guards watch real
work.  (The DuoAttention card, section Summary, fixes the cache extents these
writes must respect: sink + recent slots per streaming head.)"""
import numpy as np
import pytest
import torch

import oracle
import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs

from gpu_helpers import assert_close, host_cache, layers
from guards import Guarded

pytestmark = pytest.mark.gpu

MASK = (1, 0, 0, 1, 0, 1, 1, 0)


def fill_cache(cache, seq_len, ring_head, seed):
    for i, t in enumerate((cache.full_k, cache.full_v, cache.strm_k, cache.strm_v)):
        if t is not None:
            inputs.randn_bf16_into(t, seed * 10 + i)
    cache.seq_len.copy_(torch.as_tensor(seq_len, dtype=torch.int32))
    cache.ring_head.copy_(torch.as_tensor(ring_head, dtype=torch.int32))


@pytest.mark.parametrize("L", [129, 600])
@pytest.mark.parametrize("kind", ["duo", "sliding_gated"])
def test_prefill_writes_stay_inside(cuda_device, L, kind):
    B = 2
    g = Guarded()
    if kind == "duo":
        p, o = layers(B, full_mask=MASK)
        gate = None
    else:
        p, o = layers(B, window=512, sink_logit=inputs.randn_f32((48,), 31))
        gate = g.like(inputs.randn_bf16((B, L, 48, 128), 32, "cuda"), "gate")
    q = g.like(inputs.randn_bf16((B, L, 48, 128), 33, "cuda"), "q")
    k = g.like(inputs.randn_bf16((B, L, 8, 128), 34, "cuda"), "k")
    v = g.like(inputs.randn_bf16((B, L, 8, 128), 35, "cuda"), "v")
    out = g.empty((B, L, 48, 128), torch.bfloat16, "out", float("nan"))
    lse = g.empty((B, 48, L), torch.float32, "lse", float("nan"))
    ws = g.empty((duo.duo_prefill_workspace_bytes(),), torch.uint8, "workspace", 0x7F)
    duo.duo_attn_prefill(p, q, k, v, out, lse, workspace=ws, gate=gate)
    g.check()
    assert duo.duo_get_device_status() == duo.DUO_OK
    ro, rl = oracle.attn_prefill(o, inputs.bits(q), inputs.bits(k), inputs.bits(v))
    if gate is not None:
        ro = oracle.gate_prefill(ro, inputs.bits(gate), oracle.GATE_PER_ELEMENT, L, 48)
    assert_close(out.permute(0, 2, 1, 3).reshape(-1, 128), ro, lse.reshape(-1), rl, f"{kind} L={L}")


@pytest.mark.parametrize("kind,chunks", [("duo", [1000, 99, 1]), ("sliding", [2000, 513, 1]),
                                         ("duo_to_capacity", [700, 500])])
def test_append_writes_stay_inside(cuda_device, kind, chunks):
    B = 2
    g = Guarded()
    if kind == "sliding":
        p, o = layers(B, window=512)
    else:
        p, o = layers(B, full_mask=MASK)
    capacity = 1100 if kind == "duo_to_capacity" else 1200
    cache = g.cache(p, capacity)
    fill_cache(cache, [0, 3], [0, 7 % p.ring_slots], seed=40)
    ref = host_cache(o, cache)
    for i, n in enumerate(chunks):
        k = g.like(inputs.randn_bf16((B, n, 8, 128), 41 + 2 * i, "cuda"), f"k{i}")
        v = g.like(inputs.randn_bf16((B, n, 8, 128), 42 + 2 * i, "cuda"), f"v{i}")
        duo.duo_kv_append(p, cache, k, v)
        past = p.n_full and int(ref.seq_len.max()) + n > capacity
        if past:
            # the append stops at the capacity: compare sequence by sequence,
            # since the oracle stops at the first sequence that reaches it
            for b in range(B):
                ob = oracle.Layer(1, 48, 8, 128, o.sink, o.recent, o.window, o.softmax_scale,
                                  o.full_mask, None)
                rb = oracle.Cache(ob, capacity)
                for name in ("full_k", "full_v", "strm_k", "strm_v", "seq_len", "ring_head"):
                    setattr(rb, name, np.ascontiguousarray(getattr(ref, name)[b:b + 1]))
                kb, vb = inputs.bits(k)[b:b + 1], inputs.bits(v)[b:b + 1]
                with pytest.raises(ValueError):
                    oracle.kv_append(ob, rb, kb, vb)
                for name in ("full_k", "full_v", "strm_k", "strm_v", "seq_len", "ring_head"):
                    getattr(ref, name)[b:b + 1] = getattr(rb, name)
            assert duo.duo_get_device_status() == duo.DUO_ERR_CAPACITY
        else:
            oracle.kv_append(o, ref, inputs.bits(k), inputs.bits(v))
            assert duo.duo_get_device_status() == duo.DUO_OK
        g.check()
        got = host_cache(o, cache)
        for name in ("full_k", "full_v", "strm_k", "strm_v", "seq_len", "ring_head"):
            assert np.array_equal(getattr(got, name), getattr(ref, name)), (name, i)


def test_prep_writes_stay_inside(cuda_device):
    """The fused RMSNorm + RoPE append rewrites q and k in place and fills the
    cache with the ring wrapping (ring_head 200 of 256, 400 new tokens)."""
    B, n = 2, 400
    g = Guarded()
    p, o = layers(B, full_mask=MASK)
    cache = g.cache(p, 1000)
    fill_cache(cache, [300, 64], [200, 255], seed=50)
    ref = host_cache(o, cache)
    q = g.like(inputs.randn_bf16((B, n, 48, 128), 51, "cuda"), "q")
    k = g.like(inputs.randn_bf16((B, n, 8, 128), 52, "cuda"), "k")
    v = g.like(inputs.randn_bf16((B, n, 8, 128), 53, "cuda"), "v")
    wq = g.like((1 + 0.1 * inputs.randn_f32((128,), 54)).to("cuda", torch.bfloat16), "q_norm_weight")
    wk = g.like((1 + 0.1 * inputs.randn_f32((128,), 55)).to("cuda", torch.bfloat16), "k_norm_weight")
    prep = duo.DuoQKPrep(q_norm_weight=wq, k_norm_weight=wk)
    k_in = inputs.bits(k).copy()
    duo.duo_kv_append_prep(p, cache, prep, q, k, v)
    g.check()
    assert duo.duo_get_device_status() == duo.DUO_OK
    # the cache got the prepared k (as rewritten in place) and v, by the append rule
    oracle.kv_append(o, ref, inputs.bits(k), inputs.bits(v))
    got = host_cache(o, cache)
    for name in ("full_k", "full_v", "strm_k", "strm_v", "seq_len", "ring_head"):
        assert np.array_equal(getattr(got, name), getattr(ref, name)), name
    assert not np.array_equal(inputs.bits(k), k_in)      # k was rewritten


@pytest.mark.parametrize("q_len", [8, 150])
def test_verify_block_writes_stay_inside(cuda_device, q_len):
    B = 3
    g = Guarded()
    p, o = layers(B, full_mask=MASK)
    seq = [0, 300, 2000]
    cache = g.cache(p, 2000)
    fill_cache(cache, seq, [0, 36, 100], seed=60)
    qb = g.like(inputs.randn_bf16((B, q_len, 48, 128), 61, "cuda"), "q")
    kb = g.like(inputs.randn_bf16((B, q_len, 8, 128), 62, "cuda"), "k_new")
    vb = g.like(inputs.randn_bf16((B, q_len, 8, 128), 63, "cuda"), "v_new")
    out = g.empty((B, q_len, 48, 128), torch.bfloat16, "out", float("nan"))
    lse = g.empty((B, q_len, 48), torch.float32, "lse", float("nan"))
    nbytes = duo.duo_decode_block_workspace_bytes(p, q_len, max(seq))
    ws = g.empty(((nbytes + 255) // 256 * 256,), torch.uint8, "workspace", 0x3C)
    snap = host_cache(o, cache)
    duo.duo_attn_decode_block(p, cache, qb, kb, vb, max(seq), out, lse, ws)
    g.check()
    assert duo.duo_get_device_status() == duo.DUO_OK
    ro, rl = oracle.attn_decode_block(o, snap, inputs.bits(qb), inputs.bits(kb), inputs.bits(vb))
    assert_close(out, ro.reshape(B, q_len, 48, 128), lse, rl.reshape(B, q_len, 48), "verify block")


@pytest.mark.parametrize("kind", ["duo", "sliding"])
def test_decode_writes_stay_inside(cuda_device, kind):
    """Empty sequences next to short and long ones."""
    g = Guarded()
    seq = [0, 1, 0, 700, 3000]
    B = len(seq)
    if kind == "sliding":
        p, o = layers(B, window=512, sink_logit=inputs.randn_f32((48,), 70))
    else:
        p, o = layers(B, full_mask=MASK)
    cache = g.cache(p, 3000)
    fill_cache(cache, seq, [0, 0, 0, 100 % (p.ring_slots - p.sink), 5], seed=71)
    q = g.like(inputs.randn_bf16((B, 48, 128), 72, "cuda"), "q")
    out = g.empty((B, 48, 128), torch.bfloat16, "out", float("nan"))
    lse = g.empty((B, 48), torch.float32, "lse", float("nan"))
    nbytes = duo.duo_decode_workspace_bytes(p, max(seq))
    ws = g.empty(((nbytes + 255) // 256 * 256,), torch.uint8, "workspace", 0x3C)
    duo.duo_attn_decode(p, cache, q, max(seq), out, lse, ws)
    g.check()
    assert duo.duo_get_device_status() == duo.DUO_OK
    ro, rl = oracle.attn_decode(o, host_cache(o, cache), inputs.bits(q))
    assert_close(out, ro.reshape(B, 48, 128), lse, rl.reshape(B, 48), f"decode {kind}")
