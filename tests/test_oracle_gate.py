"""Pins of the oracle's output gate (Laguna's gated attention output; the
activation is read as the logistic sigmoid).

* g = 0 halves the output exactly (sigmoid(0) = 1/2);
* sigmoid(g) + sigmoid(-g) = 1, so the gated outputs for g and -g sum to the
  ungated output;
* a per-head gate equals the per-channel gate with its value repeated;
* the logistic function matches scipy.special.expit;
* a gate that is open (+60) at exactly one (sequence, position, head, channel)
  and closed (-60) elsewhere leaves only that element, which pins the layout
  of the gate tensor against the output rows.
"""
import numpy as np
import pytest
import scipy.special

import oracle

B, L, HQ, HKV, D = 2, 5, 48, 8, 128


def layer():
    return oracle.Layer(B, HQ, HKV, D, 64, 256, 0, D ** -0.5, (1, 0, 0, 1, 0, 1, 1, 0), None)


def bits(x: np.ndarray) -> np.ndarray:
    """float values exactly representable in bf16 -> bf16 bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def rand_bits(shape, seed, scale=1.0):
    r = np.random.default_rng(seed).standard_normal(shape).astype(np.float32) * scale
    return bits(r)   # truncation to bf16 keeps the values exact in both views


@pytest.fixture(scope="module")
def prefill_out():
    q, k, v = rand_bits((B, L, HQ, D), 1), rand_bits((B, L, HKV, D), 2), rand_bits((B, L, HKV, D), 3)
    out, _ = oracle.attn_prefill(layer(), q, k, v)
    return out


def test_zero_gate_halves_the_output(prefill_out):
    g = bits(np.zeros((B, L, HQ, D), np.float32))
    gated = oracle.gate_prefill(prefill_out, g, oracle.GATE_PER_ELEMENT, L, HQ)
    assert np.array_equal(gated, prefill_out * 0.5)


def test_gate_and_its_negation_sum_to_the_ungated_output(prefill_out):
    g = rand_bits((B, L, HQ, D), 4, scale=3.0)
    neg = bits(-oracle.bf16_bits_to_f64(g).astype(np.float32))
    a = oracle.gate_prefill(prefill_out, g, oracle.GATE_PER_ELEMENT, L, HQ)
    b = oracle.gate_prefill(prefill_out, neg, oracle.GATE_PER_ELEMENT, L, HQ)
    assert np.allclose(a + b, prefill_out, rtol=0, atol=1e-14)


def test_per_head_gate_is_the_broadcast_per_channel_gate(prefill_out):
    gh = rand_bits((B, L, HQ), 5, scale=2.0)
    ge = np.repeat(gh[..., None], D, axis=-1)
    a = oracle.gate_prefill(prefill_out, gh, oracle.GATE_PER_HEAD, L, HQ)
    b = oracle.gate_prefill(prefill_out, ge, oracle.GATE_PER_ELEMENT, L, HQ)
    assert np.array_equal(a, b)


def test_sigmoid_matches_scipy_expit():
    x = np.concatenate([np.linspace(-40, 40, 2001), np.random.default_rng(6).standard_normal(1000) * 5])
    assert np.allclose(oracle.sigmoid(x), scipy.special.expit(x), rtol=1e-14, atol=1e-300)
    assert oracle.sigmoid(np.array([-1e4]))[0] == 0.0 and oracle.sigmoid(np.array([1e4]))[0] == 1.0


@pytest.mark.parametrize("where", [(0, 0, 0, 0), (1, 3, 17, 100), (1, 4, 47, 127), (0, 2, 6, 64)])
def test_single_open_gate_pins_the_layout(prefill_out, where):
    b, i, h, d = where
    g = np.full((B, L, HQ, D), -60.0, np.float32)
    g[b, i, h, d] = 60.0
    gated = oracle.gate_prefill(prefill_out, bits(g), oracle.GATE_PER_ELEMENT, L, HQ)
    row = (b * HQ + h) * L + i          # the oracle's (b, h, i) row order
    expect = np.zeros_like(prefill_out)
    expect[row, d] = prefill_out[row, d]
    assert np.allclose(gated, expect, rtol=1e-12, atol=1e-25)


@pytest.mark.parametrize("mode", [oracle.GATE_PER_ELEMENT, oracle.GATE_PER_HEAD])
def test_decode_gate_layout(mode):
    """Decode rows are b*Hq + h: open one (b, h) gate and close the rest."""
    out = np.random.default_rng(7).standard_normal((B * HQ, D))
    shape = (B, HQ, D) if mode == oracle.GATE_PER_ELEMENT else (B, HQ)
    g = np.full(shape, -60.0, np.float32)
    g[1, 30] = 60.0
    gated = oracle.gate_decode(out, bits(g), mode, HQ)
    expect = np.zeros_like(out)
    expect[1 * HQ + 30] = out[1 * HQ + 30]
    assert np.allclose(gated, expect, rtol=1e-12, atol=1e-25)
