"""RoPE frequency tables for the configuration's optional `rope_theta`.

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
