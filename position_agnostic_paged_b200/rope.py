"""Position-encoding tables for the configuration: RoPE frequencies (`rope_theta`) and ALiBi head
slopes (`alibi_slopes`).

The kernels take their rotation frequencies from one host table per call:
theta_i = base^(-2i/d) by default, or any table passed as `Cfg.rope_theta`.
The deferred rotation itself does not change: every angle is a position
difference times theta_i.
"""
from __future__ import annotations

import math


def default_theta(base: float = 500000.0, head_dim: int = 128) -> tuple[float, ...]:
    """theta_i = base^(-2i/head_dim) for the rotate-half pairs (i, i + head_dim/2)."""
    return tuple(base ** (-2.0 * i / head_dim) for i in range(head_dim // 2))


def llama31_theta(base: float = 500000.0, head_dim: int = 128, factor: float = 8.0,
                  low_freq_factor: float = 1.0, high_freq_factor: float = 4.0,
                  original_max_position: int = 8192) -> tuple[float, ...]:
    """Frequencies with Llama-3.1 scaling (the "llama3" rope type of the Llama 3.1 configuration).

    Each default frequency f has wavelength 2*pi/f.  Short wavelengths (below
    original_max_position / high_freq_factor) keep f; long ones (above
    original_max_position / low_freq_factor) use f / factor; in between the
    frequency moves linearly, in original_max_position / wavelength, from f / factor
    at low_freq_factor to f at high_freq_factor.
    """
    short_limit = original_max_position / high_freq_factor
    long_limit = original_max_position / low_freq_factor
    out = []
    for f in default_theta(base, head_dim):
        wavelength = 2.0 * math.pi / f
        if wavelength < short_limit:
            out.append(f)
        elif wavelength > long_limit:
            out.append(f / factor)
        else:
            w = (original_max_position / wavelength - low_freq_factor) / (high_freq_factor - low_freq_factor)
            out.append(w * f + (1.0 - w) * f / factor)
    return tuple(out)


def alibi_slopes(num_heads: int) -> tuple[float, ...]:
    """ALiBi head slopes (Press, Smith and Lewis, "Train Short, Test Long", 2022) for Cfg.alibi_slopes.

    With n a power of two the slopes are r, r^2, ..., r^n for r = 2^(-8/n).  Any other head count
    takes the slopes of the largest power of two p below it and tops them up with every second
    slope (the 1st, 3rd, 5th, ...) of the 2p-head sequence.
    """
    def geometric(n):
        r = 2.0 ** (-8.0 / n)
        return [r ** (k + 1) for k in range(n)]

    if num_heads <= 0:
        raise ValueError("num_heads must be positive")
    p = 1 << (num_heads.bit_length() - 1)
    return tuple(geometric(p) + geometric(2 * p)[::2][: num_heads - p])

