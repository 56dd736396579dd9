"""Position-encoding tables for the configuration: RoPE frequencies (`rope_theta`) and ALiBi head
slopes (`alibi_slopes`).

The tables are computed by the library (lazy_rope_theta, lazy_rope_theta_llama31,
lazy_alibi_slopes in include/lazy_attn.h); these functions only forward their arguments and
keep the Llama-3.1 defaults.  The kernels take their rotation frequencies from one host table
per call, so a RoPE variant is a different table, not a different kernel: every angle is a
position difference times theta_i.
"""
from __future__ import annotations

from . import lazy_attn as la


def default_theta(base: float = 500000.0, head_dim: int = 128) -> tuple[float, ...]:
    """theta_i = base^(-2i/head_dim) for the rotate-half pairs (i, i + head_dim/2)."""
    return la.rope_theta(base, head_dim)


def llama31_theta(base: float = 500000.0, head_dim: int = 128, factor: float = 8.0,
                  low_freq_factor: float = 1.0, high_freq_factor: float = 4.0,
                  original_max_position: int = 8192) -> tuple[float, ...]:
    """Frequencies with Llama-3.1 scaling (the "llama3" rope type of the Llama 3.1 configuration),
    with that configuration's constants as defaults."""
    return la.rope_theta_llama31(base, head_dim, factor, low_freq_factor, high_freq_factor,
                                 original_max_position)


def alibi_slopes(num_heads: int) -> tuple[float, ...]:
    """ALiBi head slopes (Press, Smith and Lewis, "Train Short, Test Long", 2022); raises ValueError
    for num_heads <= 0."""
    if num_heads <= 0:
        raise ValueError("num_heads must be positive")
    return la.alibi_slopes(num_heads)
