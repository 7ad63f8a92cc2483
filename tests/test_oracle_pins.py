"""Pins the float64 oracle to things other than itself (CPU only).

* attended sets against a token-by-token simulation of the caches the pages
  describe (full cache keeps everything; streaming cache keeps the first
  `sink` tokens plus the most recent `recent`; sliding keeps the last
  `window`) -- DuoAttention Laguna Adapter card, Summary / Why It Works;
  Laguna sliding-window articles;
* attended-pair counts against their closed form, with the page constants
  from tests/golden/page_constants.json;
* outputs against torch's scaled_dot_product_attention (a library routine) in
  float64 with explicit masks, GQA groups h -> h // 6;
* special cases (streaming == causal when sink + recent >= L, sliding ==
  causal when window >= L), closed forms (K == 0 gives the mean of the
  attended values and LSE = ln |S|), and invariants (unit values give unit
  rows, or 1 - sink mass; one key gives O = V);
* cache contents after appends against the same simulation, and decode
  against prefill rows of the same sequence.
"""
import json
import math
import os
from collections import deque

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from kv_cache_reduction_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")


def page_constants():
    with open(GOLDEN) as f:
        return {k: v["value"] for k, v in json.load(f).items() if not k.startswith("_")}


# ---------------------------------------------------------------- simulation
def simulate_cache_sets(kind, L, sink, recent, window):
    """Positions held by one head's cache right after token i is appended,
    for i = 0..L-1, built by pushing tokens one at a time into lists."""
    sets = []
    if kind == "full":
        held = []
        for i in range(L):
            held.append(i)
            sets.append(set(held))
    elif kind == "streaming":
        sink_part, ring = [], deque(maxlen=recent)
        for i in range(L):
            if len(sink_part) < sink:
                sink_part.append(i)
            else:
                ring.append(i)
            sets.append(set(sink_part) | set(ring))
    else:
        ring = deque(maxlen=window)
        for i in range(L):
            ring.append(i)
            sets.append(set(ring))
    return sets


def mask_matrix(kind, L, sink, recent, window):
    m = np.zeros((L, L), dtype=bool)
    for i, s in enumerate(simulate_cache_sets(kind, L, sink, recent, window)):
        m[i, sorted(s)] = True
    return m


def layer_for(kind, sink=64, recent=256, window=512, B=1, Hq=48, Hkv=8, D=128, sigma=None):
    if kind == "sliding":
        return oracle.Layer(B, Hq, Hkv, D, sink, recent, window, D ** -0.5,
                            (0,) * Hkv, sigma)
    mask = (1,) * Hkv if kind == "full" else (0,) * Hkv
    return oracle.Layer(B, Hq, Hkv, D, sink, recent, 0, D ** -0.5, mask, sigma)


# ---------------------------------------------------------------- attended sets
@pytest.mark.parametrize("kind", ["full", "streaming", "sliding"])
@pytest.mark.parametrize("sizes", [(64, 256, 512), (2, 3, 4), (0, 1, 1), (5, 1, 7), (3, 9, 2)])
@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 319, 320, 321, 600])
def test_attended_set_matches_cache_simulation(kind, sizes, L):
    sink, recent, window = sizes
    if L > 321 and sizes != (64, 256, 512):
        pytest.skip("large L only for the page sizes")
    layer = layer_for(kind, sink, recent, window, Hq=8, Hkv=8)
    expect = mask_matrix(kind, L, sink, recent, window)
    got = np.zeros((L, L), dtype=bool)
    for i in range(L):
        for j in range(L):
            got[i, j] = oracle.attended(layer, 0, i, j)
    assert np.array_equal(got, expect)


def test_pair_counts_closed_form():
    c = page_constants()
    sink, recent, window = c["sink"], c["recent"], c["window"]
    for kind, L, span in [("streaming", 16384, sink + recent), ("sliding", 32768, window),
                          ("streaming", 1024, sink + recent), ("full", 16384, None)]:
        layer = layer_for(kind, sink, recent, window, Hq=8, Hkv=8)
        want = L * (L + 1) // 2 if span is None else sum(min(i + 1, span) for i in range(L))
        assert oracle.count_pairs(layer, 0, L) == want
    # the numbers quoted for the prefill workloads
    assert oracle.count_pairs(layer_for("streaming", Hq=8, Hkv=8), 0, 16384) == 5_191_840
    assert oracle.count_pairs(layer_for("sliding", Hq=8, Hkv=8), 0, 32768) == 16_646_400


def test_page_constants_used_by_workloads():
    c = page_constants()
    assert (inputs.SINK, inputs.RECENT, inputs.WINDOW) == (c["sink"], c["recent"], c["window"])
    assert (inputs.NUM_Q_HEADS, inputs.NUM_KV_HEADS) == (c["num_q_heads"], c["num_kv_heads"])
    w = inputs.workload("stack40")
    assert w.layers == c["layers"] and len(w.full_layers) == c["full_layers"]
    assert w.layers - len(w.full_layers) == c["sliding_layers"]
    assert w.seq_len <= c["max_position_embeddings"]


# ---------------------------------------------------------------- library pins
def rand_bits(shape, seed):
    return inputs.bits(inputs.randn_bf16(shape, seed))


def to_f64(bits_):
    return inputs.from_bits(bits_).to(torch.float64)


def sdpa_reference(q, k, v, masks, scale, sigma=None):
    """torch SDPA in float64.  q [B][L][Hq][D], k/v [B][L][Hkv][D] bits;
    masks[g] is the [L][L] boolean attended matrix of KV head g.  A sink
    logit is one extra key with value 0 whose score is sigma (additive bias)."""
    Q, K, V = to_f64(q), to_f64(k), to_f64(v)
    B, L, Hq, D = Q.shape
    Hkv = K.shape[2]
    G = Hq // Hkv
    Q = Q.permute(0, 2, 1, 3)                                 # B Hq L D
    K = K.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)     # B Hq L D
    V = V.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    M = torch.stack([torch.from_numpy(masks[h // G]) for h in range(Hq)])   # Hq L L
    bias = torch.zeros((Hq, L, L), dtype=torch.float64).masked_fill(~M, float("-inf"))
    scores = torch.matmul(Q, K.transpose(-1, -2)) * scale + bias
    if sigma is not None:
        zk = torch.zeros((B, Hq, 1, D), dtype=torch.float64)
        K = torch.cat([K, zk], dim=2)
        V = torch.cat([V, zk], dim=2)
        sig = torch.as_tensor(np.asarray(sigma, dtype=np.float64)).view(Hq, 1, 1).expand(Hq, L, 1)
        bias = torch.cat([bias, sig], dim=2)
        scores = torch.cat([scores, sig.unsqueeze(0).expand(B, Hq, L, 1)], dim=3)
    out = F.scaled_dot_product_attention(Q, K, V, attn_mask=bias.unsqueeze(0), scale=scale)
    lse = torch.logsumexp(scores, dim=-1)                     # B Hq L
    return out.permute(0, 2, 1, 3).numpy(), lse.numpy()       # B L Hq D, B Hq L


def oracle_prefill_arrays(layer, q, k, v):
    out, lse = oracle.attn_prefill(layer, q, k, v)
    B, L, Hq, D = q.shape
    out = out.reshape(B, Hq, L, D).transpose(0, 2, 1, 3)
    return out, lse.reshape(B, Hq, L)


@pytest.mark.parametrize("kind,sizes,L", [
    ("full", (64, 256, 512), 37), ("streaming", (4, 5, 0), 23), ("streaming", (64, 256, 0), 400),
    ("sliding", (0, 0, 6), 29), ("sliding", (0, 0, 512), 600)])
def test_prefill_matches_sdpa(kind, sizes, L):
    sink, recent, window = sizes
    B, Hq, Hkv, D = 2, 12, 2, 32
    layer = layer_for(kind, sink, recent, window, B=B, Hq=Hq, Hkv=Hkv, D=D)
    q = rand_bits((B, L, Hq, D), 11)
    k = rand_bits((B, L, Hkv, D), 12)
    v = rand_bits((B, L, Hkv, D), 13)
    masks = [mask_matrix(kind, L, sink, recent, window)] * Hkv
    want_o, want_l = sdpa_reference(q, k, v, masks, D ** -0.5)
    got_o, got_l = oracle_prefill_arrays(layer, q, k, v)
    np.testing.assert_allclose(got_o, want_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got_l, want_l, rtol=0, atol=1e-12)


def test_prefill_mixed_heads_and_sink_match_sdpa():
    B, Hq, Hkv, D, L = 1, 24, 4, 16, 45
    sink, recent = 3, 7
    sigma = inputs.randn_f32((Hq,), 21).numpy()
    mask = (1, 0, 0, 1)
    layer = oracle.Layer(B, Hq, Hkv, D, sink, recent, 0, 0.3, mask, sigma)
    q, k, v = rand_bits((B, L, Hq, D), 22), rand_bits((B, L, Hkv, D), 23), rand_bits((B, L, Hkv, D), 24)
    masks = [mask_matrix("full" if m else "streaming", L, sink, recent, 0) for m in mask]
    want_o, want_l = sdpa_reference(q, k, v, masks, 0.3, sigma)
    got_o, got_l = oracle_prefill_arrays(layer, q, k, v)
    np.testing.assert_allclose(got_o, want_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got_l, want_l, rtol=0, atol=1e-12)


def test_gqa_grouping_uses_contiguous_groups():
    """Query head h reads KV head h // (Hq / Hkv): make only KV head 1 nonzero
    in V and check exactly query heads 6..11 see it."""
    B, Hq, Hkv, D, L = 1, 12, 2, 8, 5
    layer = oracle.Layer(B, Hq, Hkv, D, 64, 256, 0, 0.1, (1, 1))
    q, k = rand_bits((B, L, Hq, D), 31), rand_bits((B, L, Hkv, D), 32)
    vt = torch.zeros((B, L, Hkv, D), dtype=torch.bfloat16)
    vt[:, :, 1, :] = 1.0
    out, _ = oracle_prefill_arrays(layer, q, k, inputs.bits(vt))
    assert np.all(out[:, :, :6, :] == 0.0)
    np.testing.assert_allclose(out[:, :, 6:, :], 1.0, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- special cases
def test_streaming_equals_causal_when_window_covers_sequence():
    B, Hq, Hkv, D, L = 1, 12, 2, 32, 320
    q, k, v = rand_bits((B, L, Hq, D), 41), rand_bits((B, L, Hkv, D), 42), rand_bits((B, L, Hkv, D), 43)
    full = oracle_prefill_arrays(layer_for("full", B=B, Hq=Hq, Hkv=Hkv, D=D), q, k, v)
    strm = oracle_prefill_arrays(layer_for("streaming", 64, 256, B=B, Hq=Hq, Hkv=Hkv, D=D), q, k, v)
    assert np.array_equal(full[0], strm[0]) and np.array_equal(full[1], strm[1])
    # one token longer: the last row must now differ (token 64 drops out)
    q2, k2, v2 = (rand_bits((B, L + 1, Hq, D), 41), rand_bits((B, L + 1, Hkv, D), 42),
                  rand_bits((B, L + 1, Hkv, D), 43))
    full2 = oracle_prefill_arrays(layer_for("full", B=B, Hq=Hq, Hkv=Hkv, D=D), q2, k2, v2)
    strm2 = oracle_prefill_arrays(layer_for("streaming", 64, 256, B=B, Hq=Hq, Hkv=Hkv, D=D), q2, k2, v2)
    assert np.array_equal(full2[0][:, :L], strm2[0][:, :L])
    assert not np.allclose(full2[0][:, L], strm2[0][:, L])


def test_sliding_equals_causal_when_window_covers_sequence():
    B, Hq, Hkv, D, L = 1, 12, 2, 32, 100
    q, k, v = rand_bits((B, L, Hq, D), 51), rand_bits((B, L, Hkv, D), 52), rand_bits((B, L, Hkv, D), 53)
    full = oracle_prefill_arrays(layer_for("full", B=B, Hq=Hq, Hkv=Hkv, D=D), q, k, v)
    sl = oracle_prefill_arrays(layer_for("sliding", window=100, B=B, Hq=Hq, Hkv=Hkv, D=D), q, k, v)
    assert np.array_equal(full[0], sl[0]) and np.array_equal(full[1], sl[1])
    sl99 = oracle_prefill_arrays(layer_for("sliding", window=99, B=B, Hq=Hq, Hkv=Hkv, D=D), q, k, v)
    assert np.array_equal(full[0][:, :99], sl99[0][:, :99])
    assert not np.allclose(full[0][:, 99], sl99[0][:, 99])


# ---------------------------------------------------------------- closed forms and invariants
@pytest.mark.parametrize("kind", ["full", "streaming", "sliding"])
@pytest.mark.parametrize("with_sink", [False, True])
def test_zero_keys_give_mean_of_attended_values(kind, with_sink):
    B, Hq, Hkv, D, L = 1, 6, 1, 16, 50
    sink, recent, window = 3, 5, 9
    sigma = inputs.randn_f32((Hq,), 61).numpy() if with_sink else None
    layer = layer_for(kind, sink, recent, window, B=B, Hq=Hq, Hkv=Hkv, D=D, sigma=sigma)
    q = rand_bits((B, L, Hq, D), 62)
    k = np.zeros((B, L, Hkv, D), dtype=np.uint16)
    v = rand_bits((B, L, Hkv, D), 63)
    out, lse = oracle_prefill_arrays(layer, q, k, v)
    V = to_f64(v).numpy()[0, :, 0, :]
    sets = simulate_cache_sets(kind, L, sink, recent, window)
    for i, s in enumerate(sets):
        n = len(s)
        for h in range(Hq):
            extra = math.exp(sigma[h]) if with_sink else 0.0
            # all scores are 0, so every attended key weighs e^0 = 1
            want = V[sorted(s)].sum(axis=0) / (n + extra)
            np.testing.assert_allclose(out[0, i, h], want, rtol=1e-13, atol=1e-15)
            assert abs(lse[0, h, i] - math.log(n + extra)) < 1e-13


@pytest.mark.parametrize("kind", ["full", "streaming", "sliding"])
def test_unit_values_give_unit_rows_or_one_minus_sink_mass(kind):
    B, Hq, Hkv, D, L = 2, 12, 2, 16, 70
    q, k = rand_bits((B, L, Hq, D), 71), rand_bits((B, L, Hkv, D), 72)
    ones = inputs.bits(torch.ones((B, L, Hkv, D), dtype=torch.bfloat16))
    layer = layer_for(kind, 4, 20, 30, B=B, Hq=Hq, Hkv=Hkv, D=D)
    out, _ = oracle_prefill_arrays(layer, q, k, ones)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-14)
    sigma = inputs.randn_f32((Hq,), 73).numpy() * 3
    layer_s = layer_for(kind, 4, 20, 30, B=B, Hq=Hq, Hkv=Hkv, D=D, sigma=sigma)
    out_s, lse_s = oracle_prefill_arrays(layer_s, q, k, ones)
    mass = 1.0 - np.exp(sigma[None, :, None] - lse_s)          # B Hq L
    np.testing.assert_allclose(out_s, np.broadcast_to(mass.transpose(0, 2, 1)[..., None], out_s.shape),
                               rtol=1e-12, atol=1e-14)
    assert np.all(out_s < 1.0)


def test_single_key_returns_its_value():
    B, Hq, Hkv, D = 3, 12, 2, 128
    q, k, v = rand_bits((B, 1, Hq, D), 81), rand_bits((B, 1, Hkv, D), 82), rand_bits((B, 1, Hkv, D), 83)
    for kind in ("full", "streaming", "sliding"):
        out, lse = oracle_prefill_arrays(layer_for(kind, B=B, Hq=Hq, Hkv=Hkv, D=D), q, k, v)
        V = to_f64(v).numpy()
        for h in range(Hq):
            assert np.array_equal(out[:, 0, h], V[:, 0, h // 6])
        # LSE of a single score is the score itself
        Q, K = to_f64(q).numpy(), to_f64(k).numpy()
        for b in range(B):
            for h in range(Hq):
                s = (Q[b, 0, h] * K[b, 0, h // 6]).sum() * D ** -0.5
                assert abs(lse[b, h, 0] - s) < 1e-12


# ---------------------------------------------------------------- cache append and decode
def check_cache_against_simulation(layer, cache, seqs_k, n):
    """The cache must hold exactly the tokens the simulation keeps, each in
    the slot the ring rule gives, and ring_head must point at the slot that
    holds the oldest ring token once the ring is full."""
    B, Hkv = layer.batch, layer.num_kv_heads
    S, R = (0, layer.window) if layer.window else (layer.sink, layer.recent)
    fi = ri = 0
    for g in range(Hkv):
        full = layer.window == 0 and layer.full_mask[g]
        for b in range(B):
            tok = seqs_k[b, :n, g]                    # [n][D] bits of this head
            if full:
                assert np.array_equal(cache.full_k[b, fi, :n], tok)
                continue
            kind = "sliding" if layer.window else "streaming"
            kept = simulate_cache_sets(kind, n, S, R, R)[n - 1] if n else set()
            held = cache.strm_k[b, ri]
            rows = {held[s].tobytes(): s for s in range(S + R)}
            for pos in kept:
                assert tok[pos].tobytes() in rows, f"token {pos} missing"
                slot = rows[tok[pos].tobytes()]
                if pos < S:
                    assert slot == pos
                else:
                    assert S <= slot < S + R
            ring_count = min(max(n - S, 0), R)
            if ring_count == R:
                oldest = min(p for p in kept if p >= S)
                assert rows[tok[oldest].tobytes()] == S + cache.ring_head[b]
        if full:
            fi += 1
        else:
            ri += 1
    assert np.all(cache.seq_len == n)


@pytest.mark.parametrize("kind", ["duo", "sliding"])
@pytest.mark.parametrize("chunks", [[1] * 40, [13, 1, 1, 25], [40], [3, 37]])
def test_append_matches_simulation(kind, chunks):
    B, Hq, Hkv, D = 2, 12, 2, 8
    if kind == "duo":
        layer = oracle.Layer(B, Hq, Hkv, D, 4, 9, 0, 0.25, (1, 0))
    else:
        layer = oracle.Layer(B, Hq, Hkv, D, 0, 0, 11, 0.25, (0, 0))
    T = sum(chunks)
    seq_k = rand_bits((B, T, Hkv, D), 91)
    seq_v = rand_bits((B, T, Hkv, D), 92)
    cache = oracle.Cache(layer, capacity=64)
    done = 0
    for c in chunks:
        oracle.kv_append(layer, cache, seq_k[:, done:done + c], seq_v[:, done:done + c])
        done += c
        check_cache_against_simulation(layer, cache, seq_k, done)
    # bulk and token-by-token appends leave byte-identical caches
    single = oracle.Cache(layer, capacity=64)
    for t in range(T):
        oracle.kv_append(layer, single, seq_k[:, t:t + 1], seq_v[:, t:t + 1])
    for name in ("full_k", "full_v", "strm_k", "strm_v", "seq_len", "ring_head"):
        assert np.array_equal(getattr(cache, name), getattr(single, name))


@pytest.mark.parametrize("kind", ["duo", "sliding"])
@pytest.mark.parametrize("T", [1, 3, 9, 14, 30])
def test_decode_equals_last_prefill_row(kind, T):
    """Decode of the query at position T-1 against the appended cache equals
    the library SDPA row of the whole sequence (mask from the simulation)."""
    B, Hq, Hkv, D = 2, 12, 2, 32
    sigma = inputs.randn_f32((Hq,), 101).numpy() if kind == "sliding" else None
    if kind == "duo":
        layer = oracle.Layer(B, Hq, Hkv, D, 3, 6, 0, D ** -0.5, (0, 1), sigma)
        kinds = ["streaming", "full"]
        S, R, W = 3, 6, 0
    else:
        layer = oracle.Layer(B, Hq, Hkv, D, 0, 0, 7, D ** -0.5, (0, 0), sigma)
        kinds = ["sliding", "sliding"]
        S, R, W = 0, 0, 7
    q = rand_bits((B, T, Hq, D), 102)
    k, v = rand_bits((B, T, Hkv, D), 103), rand_bits((B, T, Hkv, D), 104)
    cache = oracle.Cache(layer, capacity=T)
    oracle.kv_append(layer, cache, k, v)
    out, lse = oracle.attn_decode(layer, cache, np.ascontiguousarray(q[:, T - 1]))
    masks = [mask_matrix(kd, T, S, R, W) for kd in kinds]
    want_o, want_l = sdpa_reference(q, k, v, masks, D ** -0.5, sigma)
    np.testing.assert_allclose(out.reshape(B, Hq, D), want_o[:, T - 1], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(B, Hq), want_l[:, :, T - 1], rtol=0, atol=1e-12)


def test_decode_invariant_under_ring_slot_permutation():
    B, Hq, Hkv, D = 1, 6, 1, 16
    layer = oracle.Layer(B, Hq, Hkv, D, 4, 8, 0, 0.2, (0,))
    T = 40
    k, v = rand_bits((B, T, Hkv, D), 111), rand_bits((B, T, Hkv, D), 112)
    q = rand_bits((B, Hq, D), 113)
    cache = oracle.Cache(layer, capacity=T)
    oracle.kv_append(layer, cache, k, v)
    base = oracle.attn_decode(layer, cache, q)
    perm = np.random.default_rng(5).permutation(8)
    cache.strm_k[:, :, 4:] = cache.strm_k[:, :, 4:][:, :, perm]
    cache.strm_v[:, :, 4:] = cache.strm_v[:, :, 4:][:, :, perm]
    cache.ring_head[:] = 3
    moved = oracle.attn_decode(layer, cache, q)
    np.testing.assert_allclose(moved[0], base[0], rtol=0, atol=1e-13)
    np.testing.assert_allclose(moved[1], base[1], rtol=0, atol=1e-13)


def test_decode_empty_cache():
    B, Hq, Hkv, D = 1, 6, 1, 8
    q = rand_bits((B, Hq, D), 121)
    layer = oracle.Layer(B, Hq, Hkv, D, 4, 8, 0, 0.2, (1,))
    out, lse = oracle.attn_decode(layer, oracle.Cache(layer, 4), q)
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    sigma = np.arange(Hq, dtype=np.float32)
    layer_s = oracle.Layer(B, Hq, Hkv, D, 4, 8, 0, 0.2, (1,), sigma)
    out, lse = oracle.attn_decode(layer_s, oracle.Cache(layer_s, 4), q)
    assert np.all(out == 0) and np.allclose(lse, sigma)
