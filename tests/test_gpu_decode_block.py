"""duo_attn_decode_block (verify-block decode) on the GPU against the float64
oracle's block decode, which is pinned to the prefill oracle over the full
token history.

Every q_len from 1 to 8 (three operand widths: 16, 32 and 48 query rows),
sequences that are empty, below the sink, filling the ring and past it, a
sliding layer with sink logits, an output gate, and a 32768-token context.
The cache must be left untouched.  Tolerances as the one-token decode.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs

from gpu_helpers import assert_close, host_cache, layers, random_cache

pytestmark = pytest.mark.gpu


def block_case(p, o, cache, q_len, seed, max_seq_len, gate=None, gate_mode=0):
    B = p.batch
    q = inputs.randn_bf16((B, q_len, 48, 128), seed, "cuda")
    kn = inputs.randn_bf16((B, q_len, 8, 128), seed + 1, "cuda")
    vn = inputs.randn_bf16((B, q_len, 8, 128), seed + 2, "cuda")
    out = torch.full((B, q_len, 48, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, q_len, 48), float("nan"), dtype=torch.float32, device="cuda")
    n = max(duo.duo_decode_block_workspace_bytes(p, q_len, max_seq_len), 256)
    ws = torch.full(((n + 255) // 256 * 256,), 0x7f, dtype=torch.uint8, device="cuda")
    before = [t.clone() for t in (cache.seq_len, cache.ring_head)]
    snap = host_cache(o, cache)
    duo.duo_attn_decode_block(p, cache, q, kn, vn, max_seq_len, out, lse, ws, gate=gate)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    assert torch.equal(before[0], cache.seq_len) and torch.equal(before[1], cache.ring_head)
    after = host_cache(o, cache)
    for name in ("full_k", "full_v", "strm_k", "strm_v"):
        assert np.array_equal(getattr(after, name), getattr(snap, name)), name
    ref_o, ref_l = oracle.attn_decode_block(o, snap, inputs.bits(q), inputs.bits(kn), inputs.bits(vn))
    if gate is not None:
        ref_o = oracle.gate_decode(ref_o, inputs.bits(gate).reshape(B * q_len, 48, -1).squeeze(-1)
                                   if gate_mode == oracle.GATE_PER_HEAD else
                                   inputs.bits(gate).reshape(B * q_len, 48, 128), gate_mode, 48)
    return assert_close(out, ref_o.reshape(B, q_len, 48, 128), lse, ref_l.reshape(B, q_len, 48),
                        f"q_len={q_len}")


@pytest.mark.parametrize("q_len", [1, 2, 3, 4, 5, 6, 7, 8])
def test_block_decode_duo_layer(cuda_device, q_len):
    p, o = layers(6, full_mask=(1, 0, 0, 1, 0, 1, 1, 0))
    seq = [0, 5, 64, 200, 320, 3000]
    rh = [0, 0, 0, 136, 0, 77]
    cache = random_cache(p, 3000, seq, rh, seed=80 + q_len)
    block_case(p, o, cache, q_len, seed=90 + q_len, max_seq_len=3000)


@pytest.mark.parametrize("q_len", [4, 8])
def test_block_decode_sliding_layer_with_sink(cuda_device, q_len):
    sig = inputs.randn_f32((48,), 100)
    p, o = layers(3, window=512, sink_logit=sig)
    seq = [3, 511, 9000]
    cache = random_cache(p, 64, seq, [0, 0, 300], seed=101)
    block_case(p, o, cache, q_len, seed=102, max_seq_len=9000)


@pytest.mark.parametrize("mode", ["per_element", "per_head"])
def test_block_decode_output_gate(cuda_device, mode):
    p, o = layers(2, full_mask=(0, 1, 0, 0, 0, 0, 1, 0))
    cache = random_cache(p, 700, [700, 33], [10, 0], seed=103)
    shape = (2, 3, 48, 128) if mode == "per_element" else (2, 3, 48)
    g = (inputs.randn_f32(shape, 104) * 2.0).to("cuda", torch.bfloat16)
    gm = oracle.GATE_PER_ELEMENT if mode == "per_element" else oracle.GATE_PER_HEAD
    block_case(p, o, cache, 3, seed=105, max_seq_len=700, gate=g, gate_mode=gm)


@pytest.mark.slow
def test_block_decode_bench_shape_sampled(cuda_device):
    """The verify_b32 line's call: B=32, context 32768, decode_b32's head mask, a
    block of 8; every row of three sequences against the oracle, the cache
    untouched, every output finite."""
    w = inputs.workload("decode_b32")
    B, n, k = w.batch, w.seq_len, 8
    p, o = layers(B, full_mask=w.full_mask)
    rng = np.random.default_rng(106)
    cache = random_cache(p, n, [n] * B, rng.integers(0, 256, size=B).tolist(), seed=107)
    q = inputs.randn_bf16((B, k, 48, 128), 108, "cuda")
    kn = inputs.randn_bf16((B, k, 8, 128), 109, "cuda")
    vn = inputs.randn_bf16((B, k, 8, 128), 110, "cuda")
    out = torch.full((B, k, 48, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, k, 48), float("nan"), dtype=torch.float32, device="cuda")
    nb = duo.duo_decode_block_workspace_bytes(p, k, n)
    ws = torch.full(((nb + 255) // 256 * 256,), 0x7f, dtype=torch.uint8, device="cuda")
    before = (cache.seq_len.clone(), cache.ring_head.clone(), cache.full_k[0, 0, :64].clone(),
              cache.strm_v[B - 1, 0].clone())
    duo.duo_attn_decode_block(p, cache, q, kn, vn, n, out, lse, ws)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    assert torch.equal(before[0], cache.seq_len) and torch.equal(before[1], cache.ring_head)
    assert torch.equal(before[2], cache.full_k[0, 0, :64]) and torch.equal(before[3], cache.strm_v[B - 1, 0])
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    snap = host_cache(o, cache)
    seqs = (0, 17, 31)
    rows = [(b * k + t) * 48 + h for b in seqs for t in range(k) for h in range(48)]
    ref_o, ref_l = oracle.attn_decode_block(o, snap, inputs.bits(q), inputs.bits(kn), inputs.bits(vn),
                                            rows=rows)
    got_o = out[list(seqs)].reshape(-1, 128)
    got_l = lse[list(seqs)].reshape(-1)
    assert_close(got_o, ref_o, got_l, ref_l, "verify_b32 shape")


def test_block_decode_rejects_empty_blocks(cuda_device):
    p, o = layers(1, full_mask=(1,) * 8)
    cache = random_cache(p, 64, [10], [0], seed=109)
    q = torch.zeros((1, 1, 48, 128), dtype=torch.bfloat16, device="cuda")
    lib = duo.load_library()
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    pc, cc = p.as_c(), cache.as_c(p)
    rc = lib.duo_attn_decode_block(ctypes.byref(pc), ctypes.byref(cc), q.data_ptr(), q.data_ptr(),
                                   q.data_ptr(), 0, 64, q.data_ptr(), None, ws.data_ptr(), ws.numel(), None,
                                   None)
    assert rc == duo.DUO_ERR_UNSUPPORTED
    assert duo.duo_decode_block_workspace_bytes(p, 0, 64) == 0
    assert duo.duo_decode_block_workspace_bytes(p, 9, 64) > 0


def test_block_decode_repeat_is_bitwise_stable(cuda_device):
    """Many short items (empty, one-tile and split sequences): 40 calls on the same
    inputs give identical bytes, the first one matching the oracle.  A hand-off
    between the kernel's warps that reads a buffer one phase early shows up as a
    call that differs."""
    p, o = layers(8, full_mask=(1, 0, 0, 1, 0, 1, 1, 0))
    seq = [0, 3, 64, 130, 200, 320, 700, 2100]
    rh = [0, 0, 0, 0, 136, 0, 50, 77]
    cache = random_cache(p, 2100, seq, rh, seed=71)
    q_len = 2
    block_case(p, o, cache, q_len, seed=72, max_seq_len=2100)     # inputs from seeds 72, 73, 74
    B = p.batch
    q = inputs.randn_bf16((B, q_len, 48, 128), 72, "cuda")
    kn = inputs.randn_bf16((B, q_len, 8, 128), 73, "cuda")
    vn = inputs.randn_bf16((B, q_len, 8, 128), 74, "cuda")
    n = max(duo.duo_decode_block_workspace_bytes(p, q_len, 2100), 256)
    ws = torch.empty(((n + 255) // 256 * 256,), dtype=torch.uint8, device="cuda")
    ref_out = torch.empty((B, q_len, 48, 128), dtype=torch.bfloat16, device="cuda")
    ref_lse = torch.empty((B, q_len, 48), dtype=torch.float32, device="cuda")
    duo.duo_attn_decode_block(p, cache, q, kn, vn, 2100, ref_out, ref_lse, ws)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    out = torch.empty_like(ref_out)
    lse = torch.empty_like(ref_lse)
    for i in range(40):
        duo.duo_attn_decode_block(p, cache, q, kn, vn, 2100, out, lse, ws)
        torch.cuda.synchronize()
        assert duo.duo_get_device_status() == duo.DUO_OK
        assert torch.equal(out, ref_out), f"call {i}: output differs"
        assert torch.equal(lse, ref_lse), f"call {i}: lse differs"


# ---------------------------------------------------------------- long blocks
# q_len > 8: chunked prefill.  The two-pass path (prefill over the cached keys,
# prefill over the block's own keys, folded by their log-sum-exps) against the
# same oracle.

@pytest.mark.parametrize("q_len", [9, 130, 300])
def test_long_block_duo_layer(cuda_device, q_len):
    p, o = layers(6, full_mask=(1, 0, 0, 1, 0, 1, 1, 0))
    seq = [0, 5, 64, 200, 320, 3000]
    rh = [0, 0, 0, 136, 0, 77]
    cache = random_cache(p, 3000, seq, rh, seed=180 + q_len)
    block_case(p, o, cache, q_len, seed=190 + q_len, max_seq_len=3000)


def test_long_block_repeat_is_bitwise_stable(cuda_device):
    """The two passes of a long block share the SMs (the pass over the block's
    own keys is a programmatic dependent launch of the pass over the cached
    keys) and the fold reads both: 30 calls on the same inputs give identical
    bytes, the first one matching the oracle.  A fold that read a slice before
    its pass had written it shows up as a call that differs."""
    p, o = layers(4, full_mask=(1, 0, 0, 1, 0, 1, 1, 0))
    seq, rh = [0, 320, 1500, 3000], [0, 0, 99, 77]
    cache = random_cache(p, 3000, seq, rh, seed=214)
    q_len = 300
    block_case(p, o, cache, q_len, seed=215, max_seq_len=3000)     # inputs from seeds 215, 216, 217
    B = p.batch
    q = inputs.randn_bf16((B, q_len, 48, 128), 215, "cuda")
    kn = inputs.randn_bf16((B, q_len, 8, 128), 216, "cuda")
    vn = inputs.randn_bf16((B, q_len, 8, 128), 217, "cuda")
    n = duo.duo_decode_block_workspace_bytes(p, q_len, 3000)
    ws = torch.empty(((n + 255) // 256 * 256,), dtype=torch.uint8, device="cuda")
    ref_out = torch.empty((B, q_len, 48, 128), dtype=torch.bfloat16, device="cuda")
    ref_lse = torch.empty((B, q_len, 48), dtype=torch.float32, device="cuda")
    duo.duo_attn_decode_block(p, cache, q, kn, vn, 3000, ref_out, ref_lse, ws)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    out = torch.empty_like(ref_out)
    lse = torch.empty_like(ref_lse)
    for i in range(30):
        duo.duo_attn_decode_block(p, cache, q, kn, vn, 3000, out, lse, ws)
        torch.cuda.synchronize()
        assert duo.duo_get_device_status() == duo.DUO_OK
        assert torch.equal(out, ref_out), f"call {i}: output differs"
        assert torch.equal(lse, ref_lse), f"call {i}: lse differs"


@pytest.mark.parametrize("q_len", [200, 700])
def test_long_block_sliding_layer_with_sink(cuda_device, q_len):
    sig = inputs.randn_f32((48,), 200)
    p, o = layers(3, window=512, sink_logit=sig)
    seq = [3, 511, 9000]
    cache = random_cache(p, 64, seq, [0, 0, 300], seed=201)
    block_case(p, o, cache, q_len, seed=202 + q_len, max_seq_len=9000)


@pytest.mark.parametrize("mode", ["per_element", "per_head"])
def test_long_block_output_gate(cuda_device, mode):
    p, o = layers(2, full_mask=(0, 1, 0, 0, 0, 0, 1, 0))
    cache = random_cache(p, 700, [700, 33], [10, 0], seed=203)
    shape = (2, 150, 48, 128) if mode == "per_element" else (2, 150, 48)
    g = (inputs.randn_f32(shape, 204) * 2.0).to("cuda", torch.bfloat16)
    gm = oracle.GATE_PER_ELEMENT if mode == "per_element" else oracle.GATE_PER_HEAD
    block_case(p, o, cache, 150, seed=205, max_seq_len=700, gate=g, gate_mode=gm)


def test_long_block_ignores_unwritten_cache_memory(cuda_device):
    """Cache rows past a sequence's tokens and ring slots that hold no token are
    filled with NaN: the long path must never let them reach an output (their V
    rows are zeroed before the PV product, their scores masked)."""
    p, o = layers(3, full_mask=(1, 0, 0, 0, 0, 0, 1, 0))
    seq, rh = [0, 40, 300], [0, 0, 17]
    cache = random_cache(p, 512, seq, rh, seed=206)
    nan = float("nan")
    S, R = 64, 256
    for b, n in enumerate(seq):
        cache.full_k[b, :, n:] = nan
        cache.full_v[b, :, n:] = nan
        cache.strm_k[b, :, min(n, S):S] = nan
        cache.strm_v[b, :, min(n, S):S] = nan
        cnt = min(max(n - S, 0), R)
        for r in range(R):
            if (rh[b] - 1 - r) % R >= cnt:
                cache.strm_k[b, :, S + r] = nan
                cache.strm_v[b, :, S + r] = nan
    block_case(p, o, cache, 140, seed=207, max_seq_len=512)


@pytest.mark.slow
def test_long_block_bench_shape_sampled(cuda_device):
    """The chunk_32k line's call: a 4096-token chunk after 28672 cached tokens,
    prefill_16k's head mask (the full heads' cached keys cut into several
    slices); every query head of 24 seeded chunk positions against the oracle,
    the cache untouched, every output finite."""
    w = inputs.workload("prefill_16k")
    n, C = 28672, 4096
    p, o = layers(1, full_mask=w.full_mask)
    cache = random_cache(p, n, [n], [141], seed=210)
    q = inputs.randn_bf16((1, C, 48, 128), 211, "cuda")
    kn = inputs.randn_bf16((1, C, 8, 128), 212, "cuda")
    vn = inputs.randn_bf16((1, C, 8, 128), 213, "cuda")
    out = torch.full((1, C, 48, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((1, C, 48), float("nan"), dtype=torch.float32, device="cuda")
    nb = duo.duo_decode_block_workspace_bytes(p, C, n)
    ws = torch.full(((nb + 255) // 256 * 256,), 0x7f, dtype=torch.uint8, device="cuda")
    before = (cache.seq_len.clone(), cache.ring_head.clone(), cache.full_k[0, 0, :64].clone())
    duo.duo_attn_decode_block(p, cache, q, kn, vn, n, out, lse, ws)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    assert torch.equal(before[0], cache.seq_len) and torch.equal(before[1], cache.ring_head)
    assert torch.equal(before[2], cache.full_k[0, 0, :64])
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    snap = host_cache(o, cache)
    pos = np.sort(np.random.default_rng(214).choice(C, size=24, replace=False))
    pos[0], pos[-1] = 0, C - 1
    rows = [int(t) * 48 + h for t in pos for h in range(48)]
    ref_o, ref_l = oracle.attn_decode_block(o, snap, inputs.bits(q), inputs.bits(kn), inputs.bits(vn), rows=rows)
    got_o = out[0, pos].reshape(-1, 128)
    got_l = lse[0, pos].reshape(-1)
    assert_close(got_o, ref_o, got_l, ref_l, "chunk_32k shape")
