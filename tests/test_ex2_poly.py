"""The prefill's FMA-pipe exponential (ex2_poly2 in csrc/ptx.cuh): 2^x as 2^n
times a degree-3 polynomial in f = x - n, |f| <= 1/2, n the nearest integer.

CPU: the polynomial's coefficients, read from the source, keep the relative
error of 2^f below 7.6e-5 on [-1/2, 1/2] (a bf16 half-ulp is 2^-9 = 1.95e-3),
checked in float64 on a dense grid against numpy's exp2; and the whole
reduction, emulated step by step in float32, stays within 8e-5 of 2^x over the
range the softmax uses (x <= 8 after the running max is subtracted, and the
clamp at -125).  The GPU test of the kernel's own results is
tests/test_gpu_ex2.py."""
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def coefficients():
    src = open(os.path.join(ROOT, "kv_cache_reduction_b200", "csrc", "ptx.cuh")).read()
    body = src[src.index("ex2_poly2"):]
    vals = {k: float(v) for k, v in re.findall(r"(kC[0-3]) = ([0-9.eE+-]+)f", body)}
    return [vals[f"kC{i}"] for i in range(4)]


def test_polynomial_relative_error_bound():
    c = coefficients()
    f = np.linspace(-0.5, 0.5, 2_000_001)
    p = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    rel = np.abs(p / np.exp2(f) - 1.0)
    assert rel.max() < 7.6e-5
    # a minimax fit spreads its error: the largest error is reached at both ends
    assert rel[0] > 0.9 * rel.max() and rel[-1] > 0.9 * rel.max()


def _emulate(x):
    """The kernel's steps in float32 (fma as a float64 product-sum rounded once)."""
    c = [np.float32(v) for v in coefficients()]
    x = np.maximum(np.float32(x), np.float32(-125.0)).astype(np.float32)
    big = np.float32(12582912.0)
    j = (x + big).astype(np.float32)
    f = (x - (j - big).astype(np.float32)).astype(np.float32)
    p = np.float32(np.float64(c[3]) * f + c[2])
    p = np.float32(np.float64(p) * f + c[1])
    p = np.float32(np.float64(p) * f + c[0])
    bits = p.view(np.uint32) + (j.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_reduction_over_the_softmax_range():
    x = np.linspace(-125.0, 8.0, 1_000_003).astype(np.float32)
    y = _emulate(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 8e-5
    # integers and half-integers (the rounding ties) are covered too
    k = np.arange(-125, 9, dtype=np.float32)
    for xs in (k, k + np.float32(0.5), k - np.float32(0.5)):
        xs = xs[(xs >= -125) & (xs <= 8)]
        assert np.abs(_emulate(xs) / np.exp2(xs.astype(np.float64)) - 1.0).max() < 8e-5


def test_clamp_keeps_masked_scores_tiny_and_positive():
    y = _emulate(np.array([-np.inf, -1e30, -300.0, -126.0], dtype=np.float32)).astype(np.float64)
    assert np.all(y > 0) and np.all(y <= 2.0 ** -124)
