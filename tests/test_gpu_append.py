"""duo_kv_append on the GPU against the oracle's sequential append: the caches,
seq_len and ring_head must match byte for byte."""
import numpy as np
import pytest
import torch

import oracle
import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs

from gpu_helpers import host_cache, layers, random_cache

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


@pytest.mark.parametrize("chunks", [[1] * 20, [1000], [64, 300, 1, 1, 700], [65], [320, 1], [3, 5000]])
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


def test_append_capacity_overflow_sets_status(cuda_device):
    p, o = layers(1, full_mask=(1,) + (0,) * 7)
    cache = random_cache(p, 8, [6], [0], seed=11)
    before = inputs.bits(cache.full_k).copy()
    k = inputs.randn_bf16((1, 4, 8, 128), 500, "cuda")
    duo.duo_kv_append(p, cache, k, k)
    assert duo.duo_get_device_status() == duo.DUO_ERR_CAPACITY
    assert duo.duo_get_device_status() == duo.DUO_OK       # reading clears it
    after = inputs.bits(cache.full_k)
    # rows 6, 7 written, nothing past the capacity
    assert np.array_equal(after[0, 0, :6], before[0, 0, :6])
    assert np.array_equal(after[0, 0, 6:8], inputs.bits(k)[0, :2, 0])


def test_append_prefill_16k_workload(cuda_device):
    """The 16384-token prefill workload's cache fill (2 of 8 heads full)."""
    w = inputs.workload("prefill_16k")
    p, o = layers(w.batch, full_mask=w.full_mask)
    cache = random_cache(p, w.seq_len, [0], [0], seed=12)
    run_and_compare(p, o, cache, [w.seq_len], seed=600)
