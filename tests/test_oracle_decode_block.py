"""Pins of the oracle's block (verify) decode: k query tokens at positions
n..n+k-1 against the cache of the first n tokens, plus the block's own keys.

* It must equal the prefill oracle's rows at those positions over the full
  token history (the prefill oracle reads every key and applies the head's
  rule to positions; the block decode reads cache slots, so the two share
  only the softmax): full, streaming and sliding heads, with and without a
  sink logit, for n below the sink, inside the ring's fill and far past it.
* k = 1 must equal "append the token, then one-token decode".
* Blocks longer than the ring and the window (chunked prefill) too: their
  later queries see none of the cached ring slots.
"""
import numpy as np
import pytest

import oracle

D, HQ, HKV = 128, 12, 2


def rand_bits(shape, seed):
    r = np.random.default_rng(seed).standard_normal(shape).astype(np.float32)
    return (r.view(np.uint32) >> 16).astype(np.uint16)


def layer(B, kind, sink, recent, window, sigma):
    mask = (1, 0) if kind == "duo" else (0, 0)
    return oracle.Layer(B, HQ, HKV, D, sink, recent, window if kind == "sliding" else 0,
                        D ** -0.5, mask, sigma)


@pytest.mark.parametrize("kind", ["duo", "sliding"])
@pytest.mark.parametrize("n,k", [(0, 3), (2, 4), (5, 1), (9, 6), (23, 8), (60, 5),
                                 (0, 20), (3, 33), (11, 17), (40, 25)])
@pytest.mark.parametrize("with_sink", [False, True])
def test_block_decode_equals_prefill_rows(kind, n, k, with_sink):
    B, sink, recent, window = 2, 4, 6, 7
    sigma = np.random.default_rng(1).standard_normal(HQ) if with_sink else None
    lay = layer(B, kind, sink, recent, window, sigma)
    L = n + k
    q = rand_bits((B, L, HQ, D), 10 + n)
    kk = rand_bits((B, L, HKV, D), 20 + n)
    vv = rand_bits((B, L, HKV, D), 30 + n)
    cache = oracle.Cache(lay, max(L, 1))
    if n:
        oracle.kv_append(lay, cache, kk[:, :n], vv[:, :n])
    out, lse = oracle.attn_decode_block(lay, cache, q[:, n:], kk[:, n:], vv[:, n:])
    # prefill rows (b*HQ + h)*L + i for i in n..L-1, in the block's (b, t, h) order
    rows = [(b * HQ + h) * L + n + t for b in range(B) for t in range(k) for h in range(HQ)]
    ref_o, ref_l = oracle.attn_prefill(lay, q, kk, vv, rows=rows)
    assert np.allclose(out, ref_o, rtol=0, atol=1e-12)
    assert np.allclose(lse, ref_l, rtol=0, atol=1e-12)


@pytest.mark.parametrize("kind", ["duo", "sliding"])
@pytest.mark.parametrize("n", [0, 3, 11, 40])
def test_single_token_block_equals_append_then_decode(kind, n):
    B = 2
    lay = layer(B, kind, 4, 6, 7, None)
    kk = rand_bits((B, n + 1, HKV, D), 40 + n)
    vv = rand_bits((B, n + 1, HKV, D), 50 + n)
    q = rand_bits((B, 1, HQ, D), 60 + n)
    cache = oracle.Cache(lay, n + 1)
    if n:
        oracle.kv_append(lay, cache, kk[:, :n], vv[:, :n])
    out, lse = oracle.attn_decode_block(lay, cache, q, kk[:, n:], vv[:, n:])
    oracle.kv_append(lay, cache, kk[:, n:], vv[:, n:])
    ref_o, ref_l = oracle.attn_decode(lay, cache, q[:, 0])
    assert np.allclose(out, ref_o, rtol=0, atol=1e-12)
    assert np.allclose(lse, ref_l, rtol=0, atol=1e-12)
