"""duo_cache_bytes (KV-cache size and active utilisation, host arithmetic):
against the bytes of the tensors DuoCache.allocate actually creates, and
against a count of the valid slots the oracle's append leaves (CPU only)."""
import numpy as np
import pytest
import torch

import oracle
import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs


def allocated_bytes(params, capacity):
    c = duo.DuoCache.allocate(params, capacity, device="cpu")
    return sum(t.numel() * t.element_size() for t in (c.full_k, c.full_v, c.strm_k, c.strm_v)
               if t is not None)


@pytest.mark.parametrize("kw", [dict(full_mask=(1, 0, 0, 1, 0, 1, 1, 0)), dict(full_mask=(0,) * 8),
                                dict(full_mask=(1,) * 8), dict(window=512, full_mask=(0,) * 8)])
@pytest.mark.parametrize("capacity", [1, 320, 4096])
def test_sizes_match_the_allocated_tensors(kw, capacity):
    p = duo.DuoParams(3, **kw)
    st = duo.duo_cache_bytes(p, capacity, capacity)
    assert st.duo_bytes == allocated_bytes(p, capacity)
    full = duo.DuoParams(3, full_mask=(1,) * 8)
    assert st.full_cache_bytes == allocated_bytes(full, capacity)


@pytest.mark.parametrize("n", [0, 1, 63, 64, 300, 320, 321, 1000])
def test_active_bytes_count_valid_slots_after_appends(n):
    """Active bytes = K+V rows that hold a token the attention may read,
    counted from the oracle's cache after n sequential appends."""
    mask = inputs.seeded_full_mask(2002, 2)
    p = duo.DuoParams(2, full_mask=mask)
    o = oracle.Layer(2, 48, 8, 128, 64, 256, 0, 128 ** -0.5, mask)
    cache = oracle.Cache(o, 1024)
    if n:
        k = inputs.bits(inputs.randn_bf16((2, n, 8, 128), 5))
        oracle.kv_append(o, cache, k, k)
    # rows written at least once (fresh caches are zero; random rows are never all zero)
    written = int((cache.full_k.reshape(-1, 128) != 0).any(axis=1).sum() +
                  (cache.strm_k.reshape(-1, 128) != 0).any(axis=1).sum())
    st = duo.duo_cache_bytes(p, 1024, n)
    assert st.active_bytes == written * 128 * 2 * 2
    assert 0.0 <= st.utilization <= 1.0


def test_duo_saves_memory_at_long_context():
    p = duo.DuoParams(16, full_mask=inputs.seeded_full_mask(2005, 2))
    st = duo.duo_cache_bytes(p, 131072, 131072)
    # 2 of 8 heads keep the whole context, the other 6 keep 320 slots
    assert st.duo_bytes == 16 * (2 * 131072 + 6 * 320) * 512
    assert st.full_cache_bytes / st.duo_bytes > 3.9
    assert st.utilization == 1.0


def test_bad_arguments():
    p = duo.DuoParams(1)
    with pytest.raises(duo.DuoError):
        duo.duo_cache_bytes(p, -1, 0)
    with pytest.raises(duo.DuoError):
        duo.duo_cache_bytes(duo.DuoParams(1, head_dim=64), 16, 1)
