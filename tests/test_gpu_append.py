"""duo_kv_append on the GPU against the oracle's sequential append: the caches,
seq_len and ring_head must match byte for byte."""
import numpy as np
import pytest
import torch

import oracle
import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs

from gpu_helpers import assert_close, host_cache, layers, random_cache

pytestmark = pytest.mark.gpu


def run_and_compare(params, o_layer, cache, chunks, seed):
    ref = host_cache(o_layer, cache)
    B, H = params.batch, params.num_kv_heads
    for i, n in enumerate(chunks):
        k = inputs.randn_bf16((B, n, H, 128), seed + 2 * i, "cuda")
        v = inputs.randn_bf16((B, n, H, 128), seed + 2 * i + 1, "cuda")
        duo.duo_kv_append(params, cache, k, v)
        oracle.kv_append(o_layer, ref, inputs.bits(k), inputs.bits(v))
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    got = host_cache(o_layer, cache)
    for name in ("full_k", "full_v", "strm_k", "strm_v", "seq_len", "ring_head"):
        assert np.array_equal(getattr(got, name), getattr(ref, name)), name


# 32 tokens x 8 KV heads is the longest append done in one launch (kv_append_small),
# 33 the shortest done by the scatter and the commit
@pytest.mark.parametrize("chunks", [[1] * 20, [1000], [64, 300, 1, 1, 700], [65], [320, 1], [3, 5000],
                                    [32, 33, 32, 1]])
def test_append_duo_layer(cuda_device, chunks):
    p, o = layers(2, full_mask=(1, 0, 0, 1, 0, 1, 1, 0))
    cache = random_cache(p, 6200, [0, 0], [0, 0], seed=7)
    run_and_compare(p, o, cache, chunks, seed=100)


@pytest.mark.parametrize("chunks", [[1] * 10, [511, 2], [513], [2000, 1, 600]])
def test_append_sliding_layer(cuda_device, chunks):
    p, o = layers(3, window=512)
    cache = random_cache(p, 1, [0, 0, 0], [0, 0, 0], seed=8)
    run_and_compare(p, o, cache, chunks, seed=200)


def test_append_prefilled_cache_random_ring_head(cuda_device):
    """Decode-style appends into caches that already hold long sequences with
    the ring write pointer at arbitrary offsets."""
    B = 4
    p, o = layers(B, full_mask=inputs.seeded_full_mask(2002, 2))
    seq = [1000, 1001, 333, 64]
    rh = [17, 255, 0, 0]
    cache = random_cache(p, 1200, seq, rh, seed=9)
    run_and_compare(p, o, cache, [1, 1, 1, 40, 1], seed=300)


def test_append_small_ring_and_no_sink(cuda_device):
    p, o = layers(2, full_mask=(0, 1, 0, 0, 0, 0, 0, 0), sink=0, recent=3)
    cache = random_cache(p, 64, [0, 5], [0, 2], seed=10)
    run_and_compare(p, o, cache, [1, 2, 7, 1, 4], seed=400)


def test_append_capacity_overflow_stops_at_capacity(cuda_device):
    """An append that would take a sequence past the full cache's capacity
    appends the positions below it, drops the rest for every head (ring heads
    included), leaves seq_len at the capacity and sets DUO_ERR_CAPACITY, as
    the oracle's token-by-token append does when it stops at the capacity.
    A decode afterwards reads only the rows below the capacity."""
    p, o = layers(1, full_mask=(1,) + (0,) * 7, sink=2, recent=3)
    cache = random_cache(p, 8, [6], [1], seed=11)
    ref = host_cache(o, cache)
    k = inputs.randn_bf16((1, 4, 8, 128), 500, "cuda")
    v = inputs.randn_bf16((1, 4, 8, 128), 501, "cuda")
    duo.duo_kv_append(p, cache, k, v)
    assert duo.duo_get_device_status() == duo.DUO_ERR_CAPACITY
    assert duo.duo_get_device_status() == duo.DUO_OK       # reading clears it
    with pytest.raises(ValueError):                        # the oracle stops at the capacity too
        oracle.kv_append(o, ref, inputs.bits(k), inputs.bits(v))
    got = host_cache(o, cache)
    for name in ("full_k", "full_v", "strm_k", "strm_v", "seq_len", "ring_head"):
        assert np.array_equal(getattr(got, name), getattr(ref, name)), name
    assert int(cache.seq_len[0]) == 8
    # a full cache takes nothing more
    duo.duo_kv_append(p, cache, k[:, :1].contiguous(), v[:, :1].contiguous())
    assert duo.duo_get_device_status() == duo.DUO_ERR_CAPACITY
    again = host_cache(o, cache)
    for name in ("full_k", "full_v", "strm_k", "strm_v", "seq_len", "ring_head"):
        assert np.array_equal(getattr(again, name), getattr(ref, name)), name
    q = inputs.randn_bf16((1, 48, 128), 502, "cuda")
    out = torch.full((1, 48, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((1, 48), float("nan"), dtype=torch.float32, device="cuda")
    duo.duo_attn_decode(p, cache, q, 8, out, lse, duo.workspace_for(p, 8))
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    ro, rl = oracle.attn_decode(o, ref, inputs.bits(q))
    assert_close(out, ro.reshape(1, 48, 128), lse, rl.reshape(1, 48), "decode at capacity")


def test_append_prefill_16k_workload(cuda_device):
    """The 16384-token prefill workload's cache fill (2 of 8 heads full)."""
    w = inputs.workload("prefill_16k")
    p, o = layers(w.batch, full_mask=w.full_mask)
    cache = random_cache(p, w.seq_len, [0], [0], seed=12)
    run_and_compare(p, o, cache, [w.seq_len], seed=600)
