"""Derivation of the 2^f polynomial used by the prefill softmax.

2^x is split as 2^j * 2^f with j the nearest integer and f in [-0.5, 0.5];
2^f is approximated by the degree-3 least-squares Chebyshev fit below
(numpy.polynomial.Chebyshev.fit on 2000 Chebyshev nodes), converted to
monomial form and rounded to fp32.  Running this file prints the
coefficients and their maximum relative error on [-0.5, 0.5].
"""
import numpy as np


def coefficients(degree: int = 3, nodes: int = 2000):
    f = np.cos(np.pi * (np.arange(nodes) + 0.5) / nodes) * 0.5
    cheb = np.polynomial.chebyshev.Chebyshev.fit(f, np.exp2(f), degree, domain=[-0.5, 0.5])
    return [np.float32(c) for c in cheb.convert(kind=np.polynomial.Polynomial).coef]


def max_relative_error(coef, samples: int = 200001) -> float:
    x = np.linspace(-0.5, 0.5, samples).astype(np.float32)
    p = np.zeros_like(x)
    for c in reversed(coef):
        p = p * x + c
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = coefficients()
    print([float(v) for v in c], max_relative_error(c))
