"""duo_kv_append_prep (RMSNorm + YaRN RoPE fused into the append) on the GPU
against the float64 oracle (oracle.prep + oracle.kv_append).

q and k are rewritten in place: each value must lie within half a bf16 ulp of
the float64 result (plus 1e-6 for the float32 arithmetic near a rounding
boundary).  The cache: V rows bit-exact, K rows within one bf16 ulp (+1e-6) of
the oracle's rounded keys, seq_len / ring_head exact.  Positions reach 10^6 so
that the phase of the slowest pairs is checked far beyond the 4096-token
original context.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import prep as oprep
import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs

from gpu_helpers import host_cache, layers, random_cache

pytestmark = pytest.mark.gpu


def f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def within_half_ulp(got: np.ndarray, ref: np.ndarray, what: str):
    ulp = np.ldexp(1.0, np.frexp(ref)[1] - 8)
    bad = np.abs(got - ref) > ulp / 2 + 1e-6
    assert not bad.any(), f"{what}: {bad.sum()} values off, worst {np.abs(got - ref)[bad].max():.3e}"


def run_case(p, o, seq, ring_head, n_new, seed, prep: duo.DuoQKPrep, weights=True, scale=2.0):
    B = p.batch
    cap = max(max(seq) + n_new, 64)
    cache = random_cache(p, cap if p.n_full else 64, seq, ring_head, seed=seed)
    before = host_cache(o, cache)
    q = (inputs.randn_f32((B, n_new, 48, 128), seed + 1) * scale).to("cuda", torch.bfloat16)
    k = (inputs.randn_f32((B, n_new, 8, 128), seed + 2) * scale).to("cuda", torch.bfloat16)
    v = inputs.randn_bf16((B, n_new, 8, 128), seed + 3, "cuda")
    if weights:
        prep.q_norm_weight = (1 + 0.2 * inputs.randn_f32((128,), seed + 4)).to("cuda", torch.bfloat16)
        prep.k_norm_weight = (1 + 0.2 * inputs.randn_f32((128,), seed + 5)).to("cuda", torch.bfloat16)
    q0, k0 = f64(q), f64(k)
    duo.duo_kv_append_prep(p, cache, prep, q, k, v)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    inv = oprep.yarn_inv_freq(prep.rope_theta, prep.rope_factor, prep.original_max_position,
                              prep.beta_fast, prep.beta_slow)
    pos = np.asarray(seq, np.float64)[:, None] + np.arange(n_new)[None, :]
    wq = None if prep.q_norm_weight is None else f64(prep.q_norm_weight)
    wk = None if prep.k_norm_weight is None else f64(prep.k_norm_weight)
    q_ref = oprep.prep_rows(q0, wq, pos, inv, prep.attention_factor, prep.rms_eps)
    k_ref = oprep.prep_rows(k0, wk, pos, inv, prep.attention_factor, prep.rms_eps)
    within_half_ulp(f64(q), q_ref, "q")
    within_half_ulp(f64(k), k_ref, "k")
    oracle.kv_append(o, before, oprep.f64_to_bf16_bits(k_ref), inputs.bits(v))
    after = host_cache(o, cache)
    assert np.array_equal(after.seq_len, before.seq_len)
    assert np.array_equal(after.ring_head, before.ring_head)
    for name in ("full_v", "strm_v"):
        assert np.array_equal(getattr(after, name), getattr(before, name)), name
    to_f = lambda b: (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)
    for name in ("full_k", "strm_k"):
        g, r = to_f(getattr(after, name)), to_f(getattr(before, name))
        ulp = np.ldexp(1.0, np.frexp(r)[1] - 8)
        assert np.all(np.abs(g - r) <= ulp + 1e-6), name


def test_prep_duo_layer_ring_wraps(cuda_device):
    p, o = layers(2, full_mask=(1, 0, 0, 1, 0, 1, 1, 0))
    run_case(p, o, [0, 300], [0, 17], 40, seed=70, prep=duo.DuoQKPrep())


def test_prep_decode_shape_one_token(cuda_device):
    p, o = layers(4, full_mask=(0, 0, 1, 0, 0, 1, 0, 0))
    run_case(p, o, [1, 63, 64, 5000], [0, 0, 0, 99], 1, seed=71, prep=duo.DuoQKPrep())


def test_prep_large_positions(cuda_device):
    p, o = layers(2, full_mask=(0,) * 8)           # ring caches only: no capacity needed
    run_case(p, o, [262000, 1000000], [5, 250], 3, seed=72, prep=duo.DuoQKPrep())


def test_prep_sliding_bulk_append_keeps_survivors(cuda_device):
    p, o = layers(2, window=512)
    run_case(p, o, [10, 600], [0, 88], 700, seed=73, prep=duo.DuoQKPrep())


def test_prep_plain_rope_unit_weights(cuda_device):
    p, o = layers(1, full_mask=(1,) * 8)
    pr = duo.DuoQKPrep(rope_theta=10000.0, rope_factor=1.0, attention_factor=0.75, rms_eps=1e-5)
    run_case(p, o, [129], [0], 200, seed=74, prep=pr, weights=False)


def test_prep_rejects_bad_parameters(cuda_device):
    p, o = layers(1, full_mask=(1,) * 8)
    cache = random_cache(p, 64, [0], [0], seed=75)
    q = torch.zeros((1, 2, 48, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 2, 8, 128), dtype=torch.bfloat16, device="cuda")
    for bad in (dict(rope_theta=1.0), dict(rope_factor=0.5), dict(original_max_position=0),
                dict(beta_slow=0.0), dict(beta_fast=0.5), dict(rms_eps=-1.0)):
        with pytest.raises(duo.DuoError) as e:
            duo.duo_kv_append_prep(p, cache, duo.DuoQKPrep(**bad), q, k, k)
        assert e.value.code == duo.DUO_ERR_INVALID_ARG, bad
    assert int(cache.seq_len[0]) == 0


@pytest.mark.slow
def test_prep_bench_shape_sampled(cuda_device):
    """The bench's prep_16k call: a 16384-token prompt on the prefill_16k layer
    (positions 0..16383), every prepared q/k row checked; the cache's full
    heads checked in a seeded sample of rows, its ring heads completely."""
    w = inputs.workload("prefill_16k")
    p, o = layers(w.batch, full_mask=w.full_mask)
    L = w.seq_len
    cache = duo.DuoCache.allocate(p, L)
    q = inputs.randn_bf16((1, L, 48, 128), 110, "cuda")
    k = inputs.randn_bf16((1, L, 8, 128), 111, "cuda")
    v = inputs.randn_bf16((1, L, 8, 128), 112, "cuda")
    pr = duo.DuoQKPrep(q_norm_weight=(1 + 0.1 * inputs.randn_f32((128,), 113)).to("cuda", torch.bfloat16),
                       k_norm_weight=(1 + 0.1 * inputs.randn_f32((128,), 114)).to("cuda", torch.bfloat16))
    q0, k0 = f64(q), f64(k)
    duo.duo_kv_append_prep(p, cache, pr, q, k, v)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    inv = oprep.yarn_inv_freq(pr.rope_theta, pr.rope_factor, pr.original_max_position, pr.beta_fast,
                              pr.beta_slow)
    pos = np.arange(L, dtype=np.float64)[None, :]
    q_ref = oprep.prep_rows(q0, f64(pr.q_norm_weight), pos, inv, 1.0, pr.rms_eps)
    k_ref = oprep.prep_rows(k0, f64(pr.k_norm_weight), pos, inv, 1.0, pr.rms_eps)
    within_half_ulp(f64(q), q_ref, "q")
    within_half_ulp(f64(k), k_ref, "k")
    # the cache holds the prepared keys: full heads at their positions, ring heads the kept tokens
    kb = oprep.f64_to_bf16_bits(k_ref)
    ref = oracle.Cache(o, L)
    oracle.kv_append(o, ref, kb, inputs.bits(v))
    got = host_cache(o, cache)
    rows = np.random.default_rng(115).integers(0, L, size=512)
    to_f = lambda b: (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)
    g, r = to_f(got.full_k[:, :, rows]), to_f(ref.full_k[:, :, rows])
    assert np.all(np.abs(g - r) <= np.ldexp(1.0, np.frexp(r)[1] - 8) + 1e-6)
    assert np.array_equal(got.full_v[:, :, rows], ref.full_v[:, :, rows])
    g, r = to_f(got.strm_k), to_f(ref.strm_k)
    assert np.all(np.abs(g - r) <= np.ldexp(1.0, np.frexp(r)[1] - 8) + 1e-6)
    assert np.array_equal(got.strm_v, ref.strm_v)
    assert np.array_equal(got.seq_len, ref.seq_len) and np.array_equal(got.ring_head, ref.ring_head)
