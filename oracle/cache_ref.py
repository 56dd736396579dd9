"""Reference block cache and cache-hit simulation (TEST INFRASTRUCTURE ONLY).

Plain Python, written independently of the library's cache (lazy_cache_*) and of its simulator, to
check them: an LRU over entries sized in blocks, and the keying policies the pages compare
(gist.science, "LazyAttention: Efficient Retrieval-Augmented Generation with Deferred Positional
Encoding", Technical Summary › Experimental Results and › Problem Statement):
  agnostic     one copy per document, reused at any offset;
  aware        copies per (document, offset); a document with a copy at any offset is reused by
               re-encoding that copy for the new offset, which stores one more copy;
  aware_exact  copies per (document, offset), reused only at the same offset;
  prefix       copies per document sequence; reuse stops at the request's first miss.
Keys are Python tuples here.
"""
from __future__ import annotations

from collections import OrderedDict


class RefLRU:
    def __init__(self, capacity_blocks: int):
        self.capacity = capacity_blocks
        self.used = 0
        self.entries: OrderedDict = OrderedDict()   # key -> size, oldest first
        self.evictions = 0

    def access(self, key, n: int) -> bool:
        """True on a hit.  A miss evicts oldest entries until n blocks are free and caches the
        entry, unless it is larger than the whole cache."""
        if key in self.entries:
            self.entries.move_to_end(key)
            return True
        if n > self.capacity:
            return False
        while self.capacity - self.used < n:
            _, size = self.entries.popitem(last=False)
            self.used -= size
            self.evictions += 1
        self.entries[key] = n
        self.used += n
        return False


def ref_simulate(policy: str, doc_tokens, requests, capacity_blocks: int, block_tokens: int = 16) -> dict:
    """Block-weighted hits and misses of a request stream under one policy (see the module text)."""
    cache = RefLRU(capacity_blocks)
    copies_at: dict = {}          # aware: document -> offsets copies were written at, oldest first
    hit_b = miss_b = 0
    for req in requests:
        offset = 0
        seq = ()
        chain_intact = True
        for d in req:
            d = int(d)
            n = -(-int(doc_tokens[d]) // block_tokens)
            seq = seq + (d,)
            if policy == "agnostic":
                hit = cache.access(("doc", d), n)
            elif policy == "aware_exact":
                hit = cache.access(("doc@", d, offset), n)
            elif policy == "aware":
                here = ("doc@", d, offset)
                if here in cache.entries:
                    hit = cache.access(here, n)
                else:
                    resident = [o for o in copies_at.get(d, ()) if ("doc@", d, o) in cache.entries]
                    hit = len(resident) > 0
                    if hit:
                        cache.access(("doc@", d, resident[-1]), n)   # the copy re-encoding reads
                    cache.access(here, n)                            # the re-encoded copy
                    copies_at[d] = resident + [offset]
            elif policy == "prefix":
                hit = cache.access(("seq",) + seq, n) and chain_intact
                chain_intact = hit
            else:
                raise ValueError(policy)
            if hit:
                hit_b += n
            else:
                miss_b += n
            offset += int(doc_tokens[d])
    return {"hit_blocks": hit_b, "miss_blocks": miss_b, "evictions": cache.evictions}
