"""Cache-hit simulation for the shared pool: position-agnostic caching against position-aware and
prefix caching under a KV byte budget, on seeded RAG request streams.

Source: gist.science, "LazyAttention: Efficient Retrieval-Augmented Generation with Deferred
Positional Encoding", Experimental Results (hit ratios at a 1 GB budget under skewed access; the
gain over prefix caching and over position-aware caching) and Problem Statement (position-aware
reuse needs an exact prefix or re-encoded copies per position, which crowd the budget).

A request places its documents back to back; each document use accesses the block cache
(lazy_cache_*) under the policy's key:
  agnostic     the document: one copy serves every position;
  aware        the document and its offset, with re-encoding: a document resident at any offset is
               a hit, and serving it at an offset it has no copy for writes a re-encoded copy there
               (one cached variant per offset it has been served at);
  aware_exact  the document and its offset, without re-encoding: only a copy made at the same
               offset can be reused;
  prefix       the document sequence up to and including it: a document is reused only if every
               document before it in the request was too (the first miss ends reuse).
The hit ratio counts blocks: hit blocks / (hit + miss blocks) over the documents' blocks.
"""
from __future__ import annotations

import hashlib

import numpy as np

from .lazy_attn import BlockCache

POLICIES = ("agnostic", "aware", "aware_exact", "prefix")


def _h(*parts: int) -> int:
    """64-bit key of a tuple of integers."""
    b = np.asarray(parts, np.int64).tobytes()
    return int.from_bytes(hashlib.blake2b(b, digest_size=8).digest(), "little")


def simulate(policy: str, doc_tokens, requests, capacity_blocks: int, block_tokens: int = 16) -> dict:
    """Runs the request stream through a block cache of capacity_blocks under one policy.

    The cache holds the residency and recency of entries; a document use counts as a hit when its
    entry is resident and, under prefix caching, every earlier document of the request was a hit.
    Every use refreshes (or writes) its entry, as a recomputed document is written back."""
    if policy not in POLICIES:
        raise ValueError(policy)
    nblk = (np.asarray(doc_tokens, np.int64) + block_tokens - 1) // block_tokens
    cache = BlockCache(capacity_blocks)
    hit_b = miss_b = 0
    variants: dict[int, list[int]] = {}      # aware: offsets a copy of the document was written at
    try:
        for req in requests:
            off = 0
            reuse = True
            chain = []
            for d in req:
                d = int(d)
                n = int(nblk[d])
                if policy == "agnostic":
                    hit, _ = cache.access(_h(0, d), n)
                elif policy == "aware_exact":
                    hit, _ = cache.access(_h(1, d, off), n)
                elif policy == "aware":
                    if cache.contains(_h(1, d, off)):
                        hit, _ = cache.access(_h(1, d, off), n)
                    else:
                        live = [o for o in variants.get(d, []) if cache.contains(_h(1, d, o))]
                        hit = bool(live)
                        if hit:                       # read the newest copy, write the re-encoded one
                            cache.access(_h(1, d, live[-1]), n)
                        cache.access(_h(1, d, off), n)
                        variants[d] = live + [off]
                else:
                    chain.append(d)
                    hit, _ = cache.access(_h(2, *chain), n)
                    hit = hit and reuse
                    reuse = hit
                if hit:
                    hit_b += n
                else:
                    miss_b += n
                off += int(doc_tokens[d])
        ev = cache.stats()["evictions"]
    finally:
        cache.close()
    tot = hit_b + miss_b
    return {"policy": policy, "capacity_blocks": int(capacity_blocks), "hit_blocks": hit_b, "miss_blocks": miss_b,
            "hit_ratio": hit_b / tot if tot else 0.0, "evictions": ev}


def kv_bytes_per_block(num_kv_heads: int = 8, head_dim: int = 128, block_tokens: int = 16) -> int:
    """K and V bytes of one pool block (bf16)."""
    return num_kv_heads * block_tokens * head_dim * 2 * 2


def compare(budget_bytes: float = 2 ** 30, alphas=(0.6, 1.0, 1.4), seed: int = 1005, n_requests: int = 20000,
            order: str = "random", **stream_kw) -> list[dict]:
    """Hit ratios of the three policies per Zipf exponent at one KV budget (Llama-3.1-8B KV
    geometry: 8 KV heads x 128, bf16), with the gains of position-agnostic caching."""
    from .workloads import cache_stream
    cap = int(budget_bytes // kv_bytes_per_block())
    rows = []
    for a in alphas:
        lens, reqs = cache_stream(seed, alpha=a, n_requests=n_requests, order=order, **stream_kw)
        res = {pol: simulate(pol, lens, reqs, cap)["hit_ratio"] for pol in POLICIES}
        gain = {f"gain_vs_{k}": round(res["agnostic"] / res[k], 2) if res[k] else None for k in POLICIES[1:]}
        rows.append({"alpha": a, "order": order, "budget_bytes": int(budget_bytes), "capacity_blocks": cap,
                     **{f"hit_ratio_{k}": round(v, 4) for k, v in res.items()}, **gain})
    return rows


def budget_sweep(budgets_gb=(0.125, 0.25, 0.5, 1, 2, 4, 8), alpha: float = 1.0, seed: int = 1005,
                 n_requests: int = 6000, **stream_kw) -> list[dict]:
    """Hit ratios of the policies across KV budgets at one Zipf exponent: how the gains of
    position-agnostic caching move with the pressure on the budget."""
    from .workloads import cache_stream
    lens, reqs = cache_stream(seed, alpha=alpha, n_requests=n_requests, **stream_kw)
    rows = []
    for gb in budgets_gb:
        cap = int(gb * 2 ** 30 // kv_bytes_per_block())
        res = {pol: simulate(pol, lens, reqs, cap)["hit_ratio"] for pol in POLICIES}
        gain = {f"gain_vs_{k}": round(res["agnostic"] / res[k], 2) if res[k] else None for k in POLICIES[1:]}
        rows.append({"alpha": alpha, "budget_bytes": int(gb * 2 ** 30), "capacity_blocks": cap,
                     **{f"hit_ratio_{k}": round(v, 4) for k, v in res.items()}, **gain})
    return rows

