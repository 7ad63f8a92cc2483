"""Shared helpers for the GPU parity tests: mirrors of device caches for the
oracle, tolerance checks, and layer builders."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs

# Output tolerance for bf16 I/O with fp32 accumulation, log-sum-exp tolerance.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def layers(batch, full_mask=(0,) * 8, window=0, sink=64, recent=256, sink_logit=None,
           hkv=8, scale=128 ** -0.5):
    """(device params, oracle layer) describing the same layer."""
    sl_dev = None if sink_logit is None else sink_logit.to("cuda", torch.float32).contiguous()
    sl_host = None if sink_logit is None else sink_logit.detach().float().cpu().numpy()
    p = duo.DuoParams(batch, 6 * hkv, hkv, 128, sink, recent, window, scale, tuple(full_mask), sl_dev)
    o = oracle.Layer(batch, 6 * hkv, hkv, 128, sink, recent, window, scale, tuple(full_mask), sl_host)
    return p, o


def host_cache(o_layer: oracle.Layer, cache: duo.DuoCache) -> oracle.Cache:
    """Host copy of a device cache, in the oracle's cache type."""
    hc = oracle.Cache(o_layer, int(cache.capacity) if o_layer.n_full else 1)
    if o_layer.n_full:
        hc.full_k = inputs.bits(cache.full_k)
        hc.full_v = inputs.bits(cache.full_v)
    if o_layer.n_ring:
        hc.strm_k = inputs.bits(cache.strm_k)
        hc.strm_v = inputs.bits(cache.strm_v)
    hc.seq_len = cache.seq_len.cpu().numpy().astype(np.int32)
    hc.ring_head = cache.ring_head.cpu().numpy().astype(np.int32)
    return hc


def random_cache(params: duo.DuoParams, capacity: int, seq_len, ring_head, seed: int) -> duo.DuoCache:
    """A device cache filled with seeded N(0,1) rows and the given state."""
    c = duo.DuoCache.allocate(params, capacity)
    for i, t in enumerate((c.full_k, c.full_v, c.strm_k, c.strm_v)):
        if t is not None:
            inputs.randn_bf16_into(t, seed * 10 + i)
    c.seq_len.copy_(torch.as_tensor(seq_len, dtype=torch.int32))
    c.ring_head.copy_(torch.as_tensor(ring_head, dtype=torch.int32))
    return c


def assert_close(out_gpu: torch.Tensor, out_ref: np.ndarray, lse_gpu=None, lse_ref=None,
                 what: str = ""):
    o = out_gpu.float().cpu().numpy().reshape(out_ref.shape).astype(np.float64)
    err = np.abs(o - out_ref)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    assert err.max() <= MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean-abs {err.mean():.3e}"
    if lse_gpu is not None:
        l = lse_gpu.float().cpu().numpy().reshape(lse_ref.shape).astype(np.float64)
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(l), fin), f"{what}: lse finiteness differs"
        d = np.abs(l[fin] - lse_ref[fin])
        assert d.size == 0 or d.max() <= LSE_ABS, f"{what}: lse max-abs {d.max():.3e}"
    return err.max(), err.mean()
