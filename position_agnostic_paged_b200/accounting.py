"""Algorithmic work of the hot path: the bytes and FLOPs the method must move or compute.

These figures are the numerators of every throughput and roofline number the
benchmark reports; they count what the method needs, not what a kernel
happens to do (masked pairs, padding and re-reads are not counted).
"""
from __future__ import annotations

import numpy as np


def decode_kv_bytes(kv_len, num_kv_heads: int, head_dim: int, elem_bytes: int = 2) -> int:
    """K and V bytes one decode step reads: every visible key and value of every request once.

    Table words, the query and the output add well under 0.1% and are left out.
    """
    return int(np.sum(np.asarray(kv_len, np.int64))) * num_kv_heads * head_dim * 2 * elem_bytes


def prefill_flops(visible_pairs: int, num_q_heads: int, head_dim: int) -> int:
    """QK^T and PV multiply-adds over visible (query, key) pairs: 2*d each, per query head."""
    return 4 * head_dim * num_q_heads * int(visible_pairs)


def k_tile_rotation_overhead(m_rows: int) -> float:
    """Extra FLOPs of rotating each K tile once per query tile of m_rows rows.

    Rotating one key element costs 3 FLOPs (two products and a sum); the tile's
    key element then serves 2*m_rows FLOPs in QK^T and its value element
    another 2*m_rows in PV, hence 3 / (4 * m_rows) (gist.science, "LazyAttention:
    Efficient Retrieval-Augmented Generation with Deferred Positional
    Encoding", Technical Summary, Prefilling).
    """
    return 3.0 / (4.0 * m_rows)


def q_segment_rotation_overhead(segment_len: int) -> float:
    """Extra FLOPs when the query tile is re-rotated once per segment instead.

    Rotating the m x d query tile costs 3*m*d FLOPs per segment, against
    4*m*d*segment_len FLOPs of QK^T and PV over that segment: 3 / (4 * L).
    """
    return 3.0 / (4.0 * segment_len)
