"""Work accounting: the one overhead figure the pages print, and hand-counted totals."""
import os

import numpy as np

from position_agnostic_paged_b200 import accounting

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rotation_overhead.txt")


def test_k_tile_rotation_overhead_matches_printed_value():
    rows = [ln.split("\t") for ln in open(GOLDEN) if ln.strip() and not ln.startswith("#")]
    for m, pct, decimals in rows:
        got = 100.0 * accounting.k_tile_rotation_overhead(int(m))
        assert round(got, int(decimals)) == float(pct)


def test_segment_rotation_is_cheaper_for_long_segments():
    assert accounting.q_segment_rotation_overhead(512) < accounting.k_tile_rotation_overhead(128)
    assert accounting.q_segment_rotation_overhead(128) == accounting.k_tile_rotation_overhead(128)


def test_hand_counted_totals():
    # decode 8B shapes: 64 requests x 4161 keys x 8 KV heads x 128 x (K+V) x 2 bytes
    assert accounting.decode_kv_bytes(np.full(64, 4161), 8, 128) == 64 * 4161 * 4096
    # prefill 8B shapes: 256 queries over 5120 document keys plus a causal 256-token chunk
    pairs = 16 * (256 * 5120 + 256 * 257 // 2)
    assert accounting.prefill_flops(pairs, 32, 128) == 16 * 32 * 512 * 1343616
