"""The 2^x polynomial the prefill softmax evaluates on the FMA pipe: its
constants in csrc/ptx.cuh are the committed fit, and the whole evaluation
(nearest-integer split, polynomial, exponent add), replayed in float32 with
numpy, stays within the fit's relative error of the exact 2^x."""
import os
import re

import numpy as np

from kv_cache_reduction_b200 import exp2_poly

PTX = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "kv_cache_reduction_b200", "csrc", "ptx.cuh")


def kernel_constants():
    text = open(PTX).read()
    return [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.eE+-]+)f;", text).group(1)))
            for i in range(4)]


def test_constants_are_the_fit():
    assert kernel_constants() == exp2_poly.coefficients()


def test_fit_error_bound():
    assert exp2_poly.max_relative_error(exp2_poly.coefficients()) < 1.1e-4


def test_range_reduced_evaluation_matches_exp2():
    c = kernel_constants()
    x = np.concatenate([np.linspace(-125, 8, 400001), np.array([-0.5, 0.5, 0.0, -1.5, 7.99])])
    x = x.astype(np.float32)
    xc = np.maximum(x, np.float32(-125))
    t = (xc + np.float32(12582912.0)).astype(np.float32)
    j = (t - np.float32(12582912.0)).astype(np.float32)
    f = (xc - j).astype(np.float32)
    assert np.all(np.abs(f) <= 0.5)
    p = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    p = p.astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    y = bits.view(np.float32).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.2e-4
