"""duo_attn_decode on the GPU against the float64 oracle.

Outputs: max-abs 2e-2, mean-abs 2e-3 (bf16 out, fp32 accumulation); LSE 1e-3.
The set of cache slots each head reads is checked exactly with uniform
attention (q = 0) over one-hot value rows.
"""
import numpy as np
import pytest
import torch

import oracle
import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs

from gpu_helpers import LSE_ABS, assert_close, host_cache, layers, random_cache

pytestmark = pytest.mark.gpu


def decode_gpu(params, cache, q, max_seq_len):
    B, Hq = params.batch, params.num_q_heads
    out = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    ws = duo.workspace_for(params, max_seq_len)
    duo.duo_attn_decode(params, cache, q, max_seq_len, out, lse, ws)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    return out, lse


def check_decode(params, o_layer, cache, seed, max_seq_len=None):
    B, Hq = params.batch, params.num_q_heads
    q = inputs.randn_bf16((B, Hq, 128), seed, "cuda")
    msl = int(cache.seq_len.max().item()) if max_seq_len is None else max_seq_len
    out, lse = decode_gpu(params, cache, q, msl)
    ref_o, ref_l = oracle.attn_decode(o_layer, host_cache(o_layer, cache), inputs.bits(q))
    return assert_close(out, ref_o.reshape(B, Hq, 128), lse, ref_l.reshape(B, Hq))


@pytest.mark.parametrize("n", [1, 2, 63, 64, 65, 300, 319, 320, 321, 1000, 4097])
def test_decode_duo_layer_lengths(cuda_device, n):
    p, o = layers(2, full_mask=(1, 0, 0, 1, 0, 1, 1, 0))
    cap = max(n, 64)
    cache = random_cache(p, cap, [0, 0], [0, 0], seed=20)
    # fill through the append kernel so that ring state is the one appends leave
    k = inputs.randn_bf16((2, n, 8, 128), 21, "cuda")
    v = inputs.randn_bf16((2, n, 8, 128), 22, "cuda")
    duo.duo_kv_append(p, cache, k, v)
    check_decode(p, o, cache, seed=23)


def test_decode_mixed_lengths_and_random_ring_heads(cuda_device):
    B = 5
    p, o = layers(B, full_mask=inputs.seeded_full_mask(2002, 2))
    seq = [1, 70, 320, 5000, 333]
    rh = [0, 3, 0, 201, 12]
    cache = random_cache(p, 5000, seq, rh, seed=24)
    check_decode(p, o, cache, seed=25, max_seq_len=5000)


@pytest.mark.parametrize("n", [1, 100, 511, 512, 513, 3000])
def test_decode_sliding_layer_with_sink_logit(cuda_device, n):
    B = 3
    sig = inputs.randn_f32((48,), 26)
    p, o = layers(B, window=512, sink_logit=sig)
    cache = random_cache(p, 1, [0] * B, [0] * B, seed=27)
    k = inputs.randn_bf16((B, n, 8, 128), 28, "cuda")
    duo.duo_kv_append(p, cache, k, inputs.randn_bf16((B, n, 8, 128), 29, "cuda"))
    check_decode(p, o, cache, seed=30)


def test_decode_all_full_and_all_streaming(cuda_device):
    for mask in [(1,) * 8, (0,) * 8]:
        p, o = layers(2, full_mask=mask)
        cache = random_cache(p, 2048, [2048, 777], [0, 100], seed=31)
        check_decode(p, o, cache, seed=32, max_seq_len=2048)


def test_decode_empty_sequence(cuda_device):
    sig = inputs.randn_f32((48,), 33)
    for s in (None, sig):
        p, o = layers(2, full_mask=(1, 0, 0, 0, 0, 0, 0, 1), sink_logit=s)
        cache = random_cache(p, 64, [0, 10], [0, 0], seed=34)
        q = inputs.randn_bf16((2, 48, 128), 35, "cuda")
        out, lse = decode_gpu(p, cache, q, 64)
        assert torch.all(out[0] == 0)
        if s is None:
            assert torch.all(torch.isneginf(lse[0]))
        else:
            assert torch.allclose(lse[0].cpu(), sig, atol=1e-5)
        ref_o, ref_l = oracle.attn_decode(o, host_cache(o, cache), inputs.bits(q))
        assert_close(out, ref_o.reshape(2, 48, 128), lse, ref_l.reshape(2, 48))


def test_decode_reads_exactly_the_valid_slots(cuda_device):
    """q = 0 makes every attended slot weigh 1/|S|.  Value rows carry a one-hot
    code of the slot (slot % 128, chunk slot // 128 selected per run), so
    O[d] * |S| is 1 exactly where slot chunk*128 + d is read."""
    B = 4
    for window, mask in [(0, (1, 0, 0, 0, 0, 0, 0, 0)), (512, (0,) * 8)]:
        p, o = layers(B, full_mask=mask, window=window)
        slots = p.ring_slots
        seq = [5, 64 + 10, 64 + 256 + 30, 1000] if window == 0 else [5, 300, 512, 900]
        rh = [0, 10, 30, 77] if window == 0 else [5, 300, 0, 388]
        for chunk in range((max(slots, max(seq)) + 127) // 128):
            cache = random_cache(p, max(seq), seq, rh, seed=36)
            for key in ("strm_v", "full_v"):
                t = getattr(cache, key)
                if t is None:
                    continue
                rows = torch.arange(t.shape[2], device="cuda")
                code = torch.zeros(t.shape[2], 128, device="cuda")
                sel = (rows // 128) == chunk
                code[sel, rows[sel] % 128] = 1.0
                t.copy_(code.to(torch.bfloat16).expand_as(t))
            q = torch.zeros((B, 48, 128), dtype=torch.bfloat16, device="cuda")
            out, lse = decode_gpu(p, cache, q, max(seq))
            hc = host_cache(o, cache)
            ref_o, ref_l = oracle.attn_decode(o, hc, inputs.bits(q))
            ref_o = ref_o.reshape(B, 48, 128)
            ref_l = ref_l.reshape(B, 48)
            size = np.exp(ref_l)                      # |S|, since every score is 0
            got = out.float().cpu().numpy() * size[..., None]
            want = ref_o * size[..., None]            # 0/1 indicator from the oracle
            assert np.array_equal(np.round(got), np.round(want))
            assert np.all(np.isin(np.round(want), [0.0, 1.0]))
            assert np.abs(lse.cpu().numpy() - ref_l).max() <= LSE_ABS


def test_decode_small_workload_end_to_end(cuda_device):
    """The single-layer workload end to end: the 1024-token prompt is
    prefilled (every one of the 48 x 1024 rows against the oracle) and
    appended, then 16 steps of append-one + decode, full heads {0,3,5,6},
    every step against the oracle."""
    w = inputs.workload("decode_small")
    p, o = layers(w.batch, full_mask=w.full_mask)
    cache = duo.DuoCache.allocate(p, w.seq_len + w.decode_steps)
    ref = host_cache(o, cache)
    qp = inputs.randn_bf16((1, w.seq_len, 48, 128), w.seed + 2, "cuda")
    k = inputs.randn_bf16((1, w.seq_len, 8, 128), w.seed, "cuda")
    v = inputs.randn_bf16((1, w.seq_len, 8, 128), w.seed + 1, "cuda")
    out_p = torch.full((1, w.seq_len, 48, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse_p = torch.full((1, 48, w.seq_len), float("nan"), dtype=torch.float32, device="cuda")
    ws_p = torch.empty(duo.duo_prefill_workspace_bytes(), dtype=torch.uint8, device="cuda")
    duo.duo_attn_prefill(p, qp, k, v, out_p, lse_p, workspace=ws_p)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    ref_o, ref_l = oracle.attn_prefill(o, inputs.bits(qp), inputs.bits(k), inputs.bits(v))
    assert_close(out_p.permute(0, 2, 1, 3).reshape(-1, 128), ref_o, lse_p.reshape(-1), ref_l,
                 "prefill of the 1024-token prompt")
    duo.duo_kv_append(p, cache, k, v)
    oracle.kv_append(o, ref, inputs.bits(k), inputs.bits(v))
    for step in range(w.decode_steps):
        s = w.seed + 10 + 3 * step
        k1 = inputs.randn_bf16((1, 1, 8, 128), s, "cuda")
        v1 = inputs.randn_bf16((1, 1, 8, 128), s + 1, "cuda")
        q1 = inputs.randn_bf16((1, 48, 128), s + 2, "cuda")
        duo.duo_kv_append(p, cache, k1, v1)
        oracle.kv_append(o, ref, inputs.bits(k1), inputs.bits(v1))
        out, lse = decode_gpu(p, cache, q1, w.seq_len + w.decode_steps)
        ref_o, ref_l = oracle.attn_decode(o, ref, inputs.bits(q1))
        assert_close(out, ref_o.reshape(1, 48, 128), lse, ref_l.reshape(1, 48), f"step {step}")


@pytest.mark.slow
def test_decode_b32_workload_full_size(cuda_device):
    """B=32 at context 32768, 2 of 8 heads full, ring pointers at random
    offsets: every (sequence, query head) row against the oracle."""
    w = inputs.workload("decode_b32")
    p, o = layers(w.batch, full_mask=w.full_mask)
    rng = np.random.default_rng(w.seed)
    rh = rng.integers(0, 256, size=w.batch).tolist()
    cache = random_cache(p, w.seq_len, [w.seq_len] * w.batch, rh, seed=w.seed)
    check_decode(p, o, cache, seed=w.seed + 5, max_seq_len=w.seq_len)


@pytest.mark.parametrize("mode", ["per_element", "per_head"])
def test_decode_output_gate(cuda_device, mode):
    """out * sigmoid(g) applied in the split merge, against the oracle's gate."""
    B = 3
    p, o = layers(B, full_mask=(1, 0, 0, 1, 0, 1, 1, 0))
    seq = [5, 700, 3000]
    cache = random_cache(p, 3000, seq, [0, 11, 200], seed=60)
    q = inputs.randn_bf16((B, 48, 128), 61, "cuda")
    shape = (B, 48, 128) if mode == "per_element" else (B, 48)
    g = (inputs.randn_f32(shape, 62) * 2.5).to("cuda", torch.bfloat16)
    out = torch.empty((B, 48, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 48), dtype=torch.float32, device="cuda")
    duo.duo_attn_decode(p, cache, q, 3000, out, lse, duo.workspace_for(p, 3000), gate=g)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    ref_o, ref_l = oracle.attn_decode(o, host_cache(o, cache), inputs.bits(q))
    gm = oracle.GATE_PER_ELEMENT if mode == "per_element" else oracle.GATE_PER_HEAD
    ref_g = oracle.gate_decode(ref_o, inputs.bits(g), gm, 48)
    assert_close(out, ref_g.reshape(B, 48, 128), lse, ref_l.reshape(B, 48), mode)


def test_decode_repeat_is_bitwise_stable(cuda_device):
    """Split caches and single-split ring heads: 40 calls on the same inputs give
    identical bytes, the first one matching the oracle.  A hand-off between the
    kernel's warps that reads a buffer one phase early shows up as a call that
    differs."""
    B = 16
    p, o = layers(B, full_mask=(1, 0, 0, 1, 0, 1, 1, 0))
    seq = [0, 1, 65, 300, 320, 900, 2000, 4097, 6000, 8192, 129, 7, 5000, 2500, 640, 8000]
    rh = [(37 * b) % 256 for b in range(B)]
    cache = random_cache(p, 8192, seq, rh, seed=31)
    check_decode(p, o, cache, seed=32, max_seq_len=8192)
    q = inputs.randn_bf16((B, 48, 128), 32, "cuda")
    ref_out, ref_lse = decode_gpu(p, cache, q, 8192)
    for i in range(40):
        out, lse = decode_gpu(p, cache, q, 8192)
        assert torch.equal(out, ref_out), f"call {i}: output differs"
        assert torch.equal(lse, ref_lse), f"call {i}: lse differs"
