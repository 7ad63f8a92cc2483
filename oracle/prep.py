"""float64 oracle of the query/key preparation (test infrastructure).

RMSNorm of each head row, then the rotary embedding with YaRN frequencies, as
the Laguna pages describe them: the Laguna attention article (section on YaRN
dynamic RoPE) prints the full-attention layers' rope parameters (theta
500000, factor 64, original_max_position_embeddings 4096, beta_slow 1,
beta_fast 64, attention_factor 1, partial_rotary_factor 1); the Laguna XS 2.1
sliding-window article (section on its attention optimisations) says the
queries and keys are RMS-normalised before the rotary embedding.

The YaRN frequencies follow the published method ("NTK-by-parts", Peng et
al., YaRN: Efficient Context Window Extension of Large Language Models): a
rotary dimension pair i has base frequency theta^(-2i/D); pairs that complete
more than beta_fast turns over the original context keep it, pairs that
complete fewer than beta_slow turns are interpolated (frequency / factor),
and a linear ramp over i blends the two in between.  Readings (not on the
pages): the rotation pairs channel i with channel i + D/2; eps 1e-6.
"""
from __future__ import annotations

import math

import numpy as np

D = 128


def yarn_inv_freq(theta: float, factor: float, original_max: int, beta_fast: float,
                  beta_slow: float, d: int = D) -> np.ndarray:
    """Per-pair inverse frequencies [d/2] in float64."""
    i = np.arange(d // 2, dtype=np.float64)
    base = theta ** (-2.0 * i / d)

    def pair_index_for_turns(turns):
        # the pair whose wavelength fits `turns` times into the original context:
        # original_max * theta^(-2i/d) / (2 pi) = turns, solved for i
        return d * math.log(original_max / (turns * 2.0 * math.pi)) / (2.0 * math.log(theta))

    lo = max(math.floor(pair_index_for_turns(beta_fast)), 0)
    hi = min(math.ceil(pair_index_for_turns(beta_slow)), d - 1)
    if hi == lo:
        hi += 0.001
    ramp = np.clip((i - lo) / (hi - lo), 0.0, 1.0)   # 0: keep the base frequency, 1: interpolate
    return base * (1.0 - ramp) + (base / factor) * ramp


def rmsnorm(x: np.ndarray, weight, eps: float) -> np.ndarray:
    """x [..., D] float64; weight [D] float64 or None (unit)."""
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return y if weight is None else y * weight


def rotate(y: np.ndarray, positions: np.ndarray, inv_freq: np.ndarray,
           attention_factor: float) -> np.ndarray:
    """Rotary embedding of y [..., D] at positions [...] (float64)."""
    ang = positions[..., None].astype(np.float64) * inv_freq
    c, s = np.cos(ang), np.sin(ang)
    a, b = y[..., : D // 2], y[..., D // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1) * attention_factor


def prep_rows(x: np.ndarray, weight, positions: np.ndarray, inv_freq: np.ndarray,
              attention_factor: float, eps: float) -> np.ndarray:
    """RMSNorm then rotation.  x: [B][n][H][D] float64; positions [B][n]."""
    y = rmsnorm(x, weight, eps)
    return rotate(y, np.broadcast_to(positions[:, :, None], x.shape[:3]), inv_freq, attention_factor)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 to the nearest bf16 (8 significant bits, ties to even) in
    one step, for finite values in the normal range; returns the bit patterns."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)   # np.rint rounds half to even
    return (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
