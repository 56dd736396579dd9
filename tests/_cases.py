"""Small hand-shaped attention cases shared by the oracle pins and GPU parity tests.

Each case is a token store of raw bf16 keys/values plus, per request, a list
of segments (store row, logical offset, length) and query tokens with
positions.  Nothing here computes attention or rotations.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from position_agnostic_paged_b200.workloads import randn_bf16


@dataclass
class Case:
    hq: int
    hkv: int
    d: int
    base: float
    k_tok: np.ndarray
    v_tok: np.ndarray
    q_raw: np.ndarray
    cu_q: np.ndarray
    q_pos: np.ndarray
    seg_indptr: np.ndarray
    seg_src: np.ndarray
    seg_off: np.ndarray
    seg_len: np.ndarray

    def oracle_kwargs(self):
        return dict(num_q_heads=self.hq, num_kv_heads=self.hkv, rope_base=self.base,
                    q_raw=self.q_raw, cu_q=self.cu_q, q_pos=self.q_pos,
                    seg_indptr=self.seg_indptr, seg_src=self.seg_src, seg_off=self.seg_off,
                    seg_len=self.seg_len, k_tok=self.k_tok, v_tok=self.v_tok)


def make_case(seed: int, *, hq: int, hkv: int, d: int, base: float = 500000.0,
              requests, n_store: int | None = None) -> Case:
    """requests: list of (segments, query_positions); segments: list of (store_row, offset, length).

    The token store holds n_store rows (default: enough for every segment).
    """
    rng = np.random.default_rng(seed)
    if n_store is None:
        n_store = max([s[0] + s[2] for req in requests for s in req[0]] + [1])
    k_tok = randn_bf16(rng, (n_store, hkv, d))
    v_tok = randn_bf16(rng, (n_store, hkv, d))
    cu_q = [0]
    q_pos = []
    seg_indptr = [0]
    seg_src, seg_off, seg_len = [], [], []
    for segs, qp in requests:
        for (src, off, ln) in segs:
            seg_src.append(src)
            seg_off.append(off)
            seg_len.append(ln)
        seg_indptr.append(len(seg_src))
        q_pos.extend(qp)
        cu_q.append(len(q_pos))
    q_raw = randn_bf16(rng, (len(q_pos), hq, d))
    i32 = lambda a: np.asarray(a, np.int32)
    return Case(hq, hkv, d, base, k_tok, v_tok, q_raw, i32(cu_q), i32(q_pos), i32(seg_indptr),
                i32(seg_src), i32(seg_off), i32(seg_len))


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns to float64 by widening the bits into binary32 (exact)."""
    b = np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)
