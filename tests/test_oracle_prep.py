"""Pins of the oracle's query/key preparation (RMSNorm + YaRN rotary embedding).

* plain RoPE: with factor 1 the frequencies are theta^(-2i/D) for every pair;
* YaRN with the Laguna page's parameters: pairs that turn more than beta_fast
  times over the original 4096 positions keep their frequency, pairs that turn
  fewer than beta_slow times are divided by the factor (64), every pair
  strictly between is blended (strictly between the two), and frequencies fall
  monotonically (the method's definition in turns, not its formula in pair
  indices);
* the rotation equals multiplication of the complex numbers y_i + i y_(i+64)
  by exp(i p f_i) (an independent formulation), is the identity at position
  0, keeps each pair's norm, and makes query-key dot products depend only on
  the position difference (the defining property of rotary embeddings);
* RMSNorm: unit root-mean-square with unit weight and eps 0, invariance to a
  positive scale of the input, torch's own rms_norm (eps inside the root) on
  rows small enough for eps to matter, and 1/sqrt(2) for a constant row whose
  mean square equals eps;
* attention_factor scales the rotated rows;
* bf16 rounding: ties to even, and single rounding of float64 (no detour
  through float32).
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import prep

# the full-attention layers' rope parameters the Laguna attention article prints
_ROPE = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")))[
    "rope_full_attention"]["value"]
PAGE = dict(theta=_ROPE["rope_theta"], factor=_ROPE["factor"],
            original_max=_ROPE["original_max_position_embeddings"], beta_fast=_ROPE["beta_fast"],
            beta_slow=_ROPE["beta_slow"])


def test_page_rope_parameters():
    assert PAGE == dict(theta=500000.0, factor=64.0, original_max=4096, beta_fast=64.0, beta_slow=1.0)
    assert _ROPE["attention_factor"] == 1.0 and _ROPE["partial_rotary_factor"] == 1.0


def test_factor_one_is_plain_rope():
    f = prep.yarn_inv_freq(10000.0, 1.0, 4096, 32.0, 1.0)
    i = np.arange(64)
    assert np.allclose(f, 10000.0 ** (-i / 64.0), rtol=1e-15, atol=0)


def test_yarn_page_parameters_by_turns():
    f = prep.yarn_inv_freq(**PAGE)
    base = PAGE["theta"] ** (-np.arange(64) / 64.0)
    turns = PAGE["original_max"] * base / (2 * math.pi)   # full turns over the original context
    fast = turns > PAGE["beta_fast"]                      # above beta_fast: kept
    slow = turns < PAGE["beta_slow"]                      # below beta_slow: interpolated
    assert fast.sum() >= 8 and slow.sum() >= 16
    assert np.array_equal(f[fast], base[fast])
    assert np.allclose(f[slow], base[slow] / PAGE["factor"], rtol=1e-15, atol=0)
    assert np.all(np.diff(f) < 0)                         # monotone: no pair overtakes another
    mid = ~fast & ~slow                                   # every pair in between is blended
    assert mid.sum() >= 8
    assert np.all(f[mid] < base[mid]) and np.all(f[mid] > base[mid] / PAGE["factor"])


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_rotation_is_complex_multiplication():
    y = rand((3, 5, 4, 128), 1)
    pos = np.random.default_rng(2).integers(0, 300000, size=(3, 5)).astype(np.float64)
    f = prep.yarn_inv_freq(**PAGE)
    got = prep.rotate(y, np.broadcast_to(pos[:, :, None], y.shape[:3]), f, 1.0)
    z = (y[..., :64] + 1j * y[..., 64:]) * np.exp(1j * pos[:, :, None, None] * f)
    assert np.allclose(got[..., :64], z.real, rtol=0, atol=1e-12)
    assert np.allclose(got[..., 64:], z.imag, rtol=0, atol=1e-12)


def test_rotation_identity_at_zero_and_pair_norms_kept():
    y = rand((2, 3, 2, 128), 3)
    f = prep.yarn_inv_freq(**PAGE)
    zero = prep.rotate(y, np.zeros(y.shape[:3]), f, 1.0)
    assert np.array_equal(zero, y)
    pos = np.full(y.shape[:3], 12345.0)
    r = prep.rotate(y, pos, f, 1.0)
    n_in = y[..., :64] ** 2 + y[..., 64:] ** 2
    n_out = r[..., :64] ** 2 + r[..., 64:] ** 2
    assert np.allclose(n_in, n_out, rtol=1e-12, atol=0)


def test_attention_factor_scales_the_rotated_rows():
    y = rand((2, 3, 2, 128), 9)
    f = prep.yarn_inv_freq(**PAGE)
    pos = np.full(y.shape[:3], 777.0)
    assert np.allclose(prep.rotate(y, pos, f, 0.75), 0.75 * prep.rotate(y, pos, f, 1.0), rtol=1e-15, atol=0)
    assert np.allclose(prep.rotate(y, np.zeros(y.shape[:3]), f, 1.25), 1.25 * y, rtol=1e-15, atol=0)


def test_dot_products_depend_only_on_position_difference():
    q, k = rand((1, 1, 1, 128), 4), rand((1, 1, 1, 128), 5)
    f = prep.yarn_inv_freq(**PAGE)
    rot = lambda x, p: prep.rotate(x, np.full((1, 1, 1), float(p)), f, 1.0).ravel()
    ref = rot(q, 1000) @ rot(k, 700)
    for shift in (1, 77, 4096, 100000):
        assert abs(rot(q, 1000 + shift) @ rot(k, 700 + shift) - ref) < 1e-9 * max(1.0, abs(ref))


def test_rmsnorm_unit_rms_and_scale_invariance():
    x = rand((4, 128), 6, scale=7.0)
    y = prep.rmsnorm(x, None, 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-14)
    assert np.allclose(prep.rmsnorm(3.5 * x, None, 0.0), y, rtol=1e-14, atol=0)
    w = rand(128, 7)
    assert np.allclose(prep.rmsnorm(x, w, 0.0), y * w, rtol=1e-15, atol=0)


def test_rmsnorm_matches_torch_where_eps_matters():
    import torch
    x = rand((6, 128), 10, scale=2e-3)                    # mean square ~ eps
    w = 1 + 0.1 * rand(128, 11)
    want = torch.nn.functional.rms_norm(torch.from_numpy(x), (128,), torch.from_numpy(w), 1e-6)
    assert np.allclose(prep.rmsnorm(x, w, 1e-6), want.numpy(), rtol=1e-13, atol=0)
    c = np.full((1, 128), 1e-3)                           # mean square 1e-6 = eps
    assert np.allclose(prep.rmsnorm(c, None, 1e-6), 2 ** -0.5, rtol=1e-14, atol=0)


def test_bf16_rounding_ties_to_even_and_single_rounding():
    to_f = lambda b: (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1.0)
    assert prep.f64_to_bf16_bits(np.array([1.0 + 2 ** -8]))[0] == 0x3F80
    # 1 + 3 * 2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6
    assert to_f(prep.f64_to_bf16_bits(np.array([1.0 + 3 * 2 ** -8])))[0] == 1.0 + 2 ** -6
    # just below a tie in float64 but a tie after rounding to float32: stays below
    x = -2.2734374098623973
    assert to_f(prep.f64_to_bf16_bits(np.array([x])))[0] == -2.265625
    r = rand(10000, 8, scale=5.0)
    b = to_f(prep.f64_to_bf16_bits(r))
    ulp = np.ldexp(1.0, np.frexp(r)[1] - 8)
    assert np.all(np.abs(b - r) <= ulp / 2)
