"""Seeded synthetic workloads for deferred-RoPE attention over a paged KV cache.

This module only makes inputs: random bf16 tensors, document populations,
Zipf-skewed document draws, the placement of every token in the paged pool
and the logical offset of every segment.  It holds none of the method's
arithmetic (no rotation, no word packing, no attention), and both the CUDA
path and the CPU oracle read its output.

Workload shapes follow the pages' experiments: RAG requests that concatenate
retrieved documents with a question, with skewed ("hot document") access
(gist.science, "LazyAttention: Efficient Retrieval-Augmented Generation with
Deferred Positional Encoding", Technical Summary: Problem Statement and
Experimental Results), on Llama-3.1-8B/70B attention shapes.  The pages
measure on RAG QA datasets; those are not used: documents and questions here
are N(0, 1) random tensors of the same shapes.

Recipe (every draw comes from numpy PCG64 seeded per purpose):
  * document d's raw keys/values: default_rng([seed, 1, d]); request r's
    question tokens: default_rng([seed, 2, r]); request r's queries:
    default_rng([seed, 3, r]); document lengths and draws: default_rng([seed, 0]).
  * values are N(0, 1) float32 rounded to bf16 (nearest, ties to even).
  * finite Zipf: P(document of rank k) proportional to k^-alpha, k = 1..N,
    rank = document id + 1; alpha = 0 is uniform.  Draws are without
    replacement inside a request and independent across requests; the drawn
    documents are then shuffled and placed contiguously from offset 0; the
    question follows at the total document length.
  * pool placement: document d owns consecutive 16-token blocks; each
    request's question owns blocks after all documents.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import numpy as np

BLOCK = 16


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (inputs are finite)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + r) >> np.uint32(16)).astype(np.uint16)


def randn_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    return bf16_bits(rng.standard_normal(shape, dtype=np.float32))


def zipf_probs(n: int, alpha: float) -> np.ndarray:
    k = np.arange(1, n + 1, dtype=np.float64)
    w = k ** (-float(alpha))
    return w / w.sum()


@dataclass
class Step:
    """One attention launch over a batch of requests.

    kind: "prefill" (a chunk of query tokens per request, causal) or "decode"
    (one query token per request).  write_rows are the token-store rows whose
    K/V are written into the pool right before this step's attention (the
    prefill chunk itself, or the decode token).
    """
    kind: str
    write_rows: np.ndarray          # int64 [n_w]
    q_raw: np.ndarray               # uint16 [total_q, Hq, d]
    cu_q: np.ndarray                # int32 [B+1]
    q_pos: np.ndarray               # int32 [total_q] logical position of each query token
    q_pos0: np.ndarray              # int32 [B] position of each request's first query token
    table_indptr: np.ndarray        # int32 [B+1]
    table_block: np.ndarray         # int32 [n_words] physical block id per logical block
    table_off: np.ndarray           # int32 [n_words] segment logical offset per logical block
    seg_indptr: np.ndarray          # int32 [B+1]
    seg_src: np.ndarray             # int32 [n_seg] first token-store row of the segment
    seg_off: np.ndarray             # int32 [n_seg] logical offset of the segment
    seg_len: np.ndarray             # int32 [n_seg] tokens in the segment (as of this step)
    kv_len: np.ndarray              # int64 [B]
    visible_pairs: int = 0          # sum over requests and query tokens of visible keys (one head)

    @property
    def num_req(self) -> int:
        return int(self.cu_q.size - 1)

    @property
    def total_q(self) -> int:
        return int(self.cu_q[-1])

    @property
    def max_words(self) -> int:
        return int(np.diff(self.table_indptr).max()) if self.num_req else 0


@dataclass
class Workload:
    name: str
    hq: int
    hkv: int
    d: int
    rope_base: float
    num_blocks: int
    k_store: np.ndarray             # uint16 [n_store, Hkv, d] raw (unrotated) keys
    v_store: np.ndarray             # uint16 [n_store, Hkv, d]
    store_slot: np.ndarray          # int32 [n_store] pool slot = block*16 + s
    store_j: np.ndarray             # int32 [n_store] local index inside the token's segment
    setup_rows: np.ndarray          # int64: rows written before any step (documents, cached questions)
    steps: list = field(default_factory=list)
    info: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.hq // self.hkv


class _Builder:
    """Accumulates token-store rows and pool placements."""

    def __init__(self, hkv: int, d: int):
        self.hkv, self.d = hkv, d
        self.k_parts, self.v_parts, self.slot_parts, self.j_parts = [], [], [], []
        self.n = 0

    def add(self, k: np.ndarray, v: np.ndarray, first_block: int) -> int:
        """Adds a segment's tokens placed from first_block on; returns its first store row."""
        n = k.shape[0]
        j = np.arange(n, dtype=np.int64)
        self.k_parts.append(k)
        self.v_parts.append(v)
        self.slot_parts.append((first_block * BLOCK + j).astype(np.int32))
        self.j_parts.append(j.astype(np.int32))
        row = self.n
        self.n += n
        return row

    def finish(self):
        if self.n == 0:
            z = np.zeros((0, self.hkv, self.d), np.uint16)
            return z, z.copy(), np.zeros(0, np.int32), np.zeros(0, np.int32)
        return (np.concatenate(self.k_parts), np.concatenate(self.v_parts),
                np.concatenate(self.slot_parts), np.concatenate(self.j_parts))


def _blocks(n_tok: int) -> int:
    return (n_tok + BLOCK - 1) // BLOCK


def _request_tables(docs, doc_first_block, doc_len, doc_row, q_first_block, q_row, q_len, q_off):
    """Unpacked table (block, offset per logical block) and oracle segments of one request."""
    blocks, offs, segs = [], [], []
    off = 0
    for dd in docs:
        nb = _blocks(doc_len[dd])
        blocks.extend(range(doc_first_block[dd], doc_first_block[dd] + nb))
        offs.extend([off] * nb)
        segs.append((doc_row[dd], off, doc_len[dd]))
        off += doc_len[dd]
    assert off == q_off
    if q_len > 0:
        nb = _blocks(q_len)
        blocks.extend(range(q_first_block, q_first_block + nb))
        offs.extend([q_off] * nb)
        segs.append((q_row, q_off, q_len))
    return blocks, offs, segs


def _make_step(kind, write_rows, q_raw, q_pos_list, tables):
    B = len(tables)
    cu_q = np.zeros(B + 1, np.int32)
    cu_q[1:] = np.cumsum([len(p) for p in q_pos_list])
    q_pos = np.concatenate([np.asarray(p, np.int32) for p in q_pos_list]) if B else np.zeros(0, np.int32)
    q_pos0 = np.array([p[0] for p in q_pos_list], np.int32)
    t_ind = np.zeros(B + 1, np.int32)
    t_ind[1:] = np.cumsum([len(t[0]) for t in tables])
    s_ind = np.zeros(B + 1, np.int32)
    s_ind[1:] = np.cumsum([len(t[2]) for t in tables])
    tb = np.array([b for t in tables for b in t[0]], np.int32)
    to = np.array([o for t in tables for o in t[1]], np.int32)
    segs = [s for t in tables for s in t[2]]
    seg_src = np.array([s[0] for s in segs], np.int32)
    seg_off = np.array([s[1] for s in segs], np.int32)
    seg_len = np.array([s[2] for s in segs], np.int32)
    kv_len = np.array([sum(s[2] for s in t[2]) for t in tables], np.int64)
    vis = 0
    for r, t in enumerate(tables):
        pos = np.concatenate([np.arange(s[1], s[1] + s[2]) for s in t[2]]) if t[2] else np.zeros(0)
        pos = np.sort(pos)
        qp = np.asarray(q_pos_list[r])
        vis += int(np.searchsorted(pos, qp, side="right").sum())
    return Step(kind=kind, write_rows=np.asarray(write_rows, np.int64), q_raw=q_raw, cu_q=cu_q,
                q_pos=q_pos, q_pos0=q_pos0, table_indptr=t_ind, table_block=tb, table_off=to,
                seg_indptr=s_ind, seg_src=seg_src, seg_off=seg_off, seg_len=seg_len,
                kv_len=kv_len, visible_pairs=vis)


def build_rag(*, name: str, seed: int, hq: int, hkv: int, d: int = 128, rope_base: float = 500000.0,
              n_docs: int, doc_len, docs_per_req: int, alpha: float, n_prefill: int = 0,
              prefill_len: int = 256, n_decode: int = 0, question_len: int = 64,
              decode_steps: int = 1, pool_cap_blocks: int | None = None,
              prefill_docs_per_req: int | None = None, uniform_docs: bool = False,
              distinct_docs: bool = False) -> Workload:
    """General RAG workload: prefill chunks and/or decode requests over a shared pool.

    doc_len: an int (every document that long) or a (lo, hi) pair (uniform).
    Prefill requests: prefill_docs_per_req documents, then a prefill_len-token
    question chunk written in the step and queried causally.
    Decode requests: docs_per_req documents, a question_len-token question
    already cached, then decode_steps steps that each write one token and query it.
    pool_cap_blocks: if set, the pool holds at most that many blocks in total
    (questions included); the document population is the popularity-ranked
    prefix of documents that fits.
    distinct_docs: draw the documents of all requests together, without
    replacement, so that no document is shared by two requests (every logical
    K/V byte of the step is then a distinct physical byte).
    """
    rng0 = np.random.default_rng([seed, 0])
    pf_docs = prefill_docs_per_req if prefill_docs_per_req is not None else docs_per_req
    if isinstance(doc_len, (tuple, list)):
        lens = rng0.integers(doc_len[0], doc_len[1] + 1, size=n_docs).astype(np.int64)
    else:
        lens = np.full(n_docs, int(doc_len), np.int64)
    q_blocks_pf = _blocks(prefill_len)
    q_blocks_dec = _blocks(question_len + decode_steps)
    q_blocks_total = n_prefill * q_blocks_pf + n_decode * q_blocks_dec
    doc_blocks = np.array([_blocks(int(x)) for x in lens], np.int64)
    if pool_cap_blocks is not None:
        room = pool_cap_blocks - q_blocks_total
        csum = np.cumsum(doc_blocks)
        n_docs = int(np.searchsorted(csum, room, side="right"))
        lens = lens[:n_docs]
        doc_blocks = doc_blocks[:n_docs]
    assert n_docs >= max(docs_per_req if n_decode else 0, pf_docs if n_prefill else 0)
    doc_first = np.zeros(n_docs, np.int64)
    doc_first[1:] = np.cumsum(doc_blocks)[:-1]
    doc_region = int(doc_blocks.sum())
    num_blocks = pool_cap_blocks if pool_cap_blocks is not None else doc_region + q_blocks_total
    p = None if (uniform_docs or alpha == 0) else zipf_probs(n_docs, alpha)

    def draw(k):
        sel = rng0.choice(n_docs, size=k, replace=False, p=p)
        return [int(x) for x in rng0.permutation(sel)]

    if distinct_docs:
        need = n_prefill * pf_docs + n_decode * docs_per_req
        assert need <= n_docs, "distinct documents: the pool is too small"
        allsel = [int(x) for x in rng0.choice(n_docs, size=need, replace=False, p=p)]
        pf_draws = [allsel[i * pf_docs:(i + 1) * pf_docs] for i in range(n_prefill)]
        base = n_prefill * pf_docs
        dec_draws = [allsel[base + i * docs_per_req: base + (i + 1) * docs_per_req] for i in range(n_decode)]
    else:
        pf_draws = [draw(pf_docs) for _ in range(n_prefill)]
        dec_draws = [draw(docs_per_req) for _ in range(n_decode)]

    used = sorted(set(x for dd in pf_draws + dec_draws for x in dd))
    bld = _Builder(hkv, d)
    doc_row = {}
    for dd in used:
        g = np.random.default_rng([seed, 1, dd])
        L = int(lens[dd])
        k = randn_bf16(g, (L, hkv, d))
        v = randn_bf16(g, (L, hkv, d))
        doc_row[dd] = bld.add(k, v, int(doc_first[dd]))
    n_setup_docs = bld.n

    next_block = doc_region
    steps = []
    setup_extra = []
    # prefill requests: their chunk is written in the step
    if n_prefill:
        tables, qps, qraws, wrows = [], [], [], []
        for r, dd in enumerate(pf_draws):
            g = np.random.default_rng([seed, 2, r])
            k = randn_bf16(g, (prefill_len, hkv, d))
            v = randn_bf16(g, (prefill_len, hkv, d))
            q_off = int(sum(lens[x] for x in dd))
            row = bld.add(k, v, next_block)
            qb = next_block
            next_block += q_blocks_pf
            wrows.append(np.arange(row, row + prefill_len))
            tables.append(_request_tables(dd, doc_first, lens, doc_row, qb, row, prefill_len, q_off))
            qps.append(np.arange(q_off, q_off + prefill_len))
            gq = np.random.default_rng([seed, 3, r])
            qraws.append(randn_bf16(gq, (prefill_len, hq, d)))
        steps.append(_make_step("prefill", np.concatenate(wrows), np.concatenate(qraws), qps, tables))
    # decode requests: question cached at setup, then one token per step
    if n_decode:
        qrows, qfirst, qoff = [], [], []
        for r, dd in enumerate(dec_draws):
            g = np.random.default_rng([seed, 2, n_prefill + r])
            n_q = question_len + decode_steps
            k = randn_bf16(g, (n_q, hkv, d))
            v = randn_bf16(g, (n_q, hkv, d))
            row = bld.add(k, v, next_block)
            qfirst.append(next_block)
            next_block += q_blocks_dec
            qrows.append(row)
            qoff.append(int(sum(lens[x] for x in dd)))
            setup_extra.append(np.arange(row, row + question_len))
        for st in range(decode_steps):
            tables, qps, qraws, wrows = [], [], [], []
            for r, dd in enumerate(dec_draws):
                cached = question_len + st + 1
                wrows.append(qrows[r] + question_len + st)
                tables.append(_request_tables(dd, doc_first, lens, doc_row, qfirst[r], qrows[r],
                                              cached, qoff[r]))
                qps.append([qoff[r] + question_len + st])
                gq = np.random.default_rng([seed, 3, n_prefill + r, st])
                qraws.append(randn_bf16(gq, (1, hq, d)))
            steps.append(_make_step("decode", np.array(wrows), np.concatenate(qraws), qps, tables))
    assert next_block <= num_blocks
    k_store, v_store, slot, j = bld.finish()
    setup_rows = np.concatenate([np.arange(n_setup_docs)] + setup_extra).astype(np.int64)
    info = dict(n_docs=n_docs, unique_docs_used=len(used), doc_region_blocks=doc_region,
                alpha=alpha, seed=seed)
    return Workload(name=name, hq=hq, hkv=hkv, d=d, rope_base=rope_base, num_blocks=int(num_blocks),
                    k_store=k_store, v_store=v_store, store_slot=slot, store_j=j,
                    setup_rows=setup_rows, steps=steps, info=info)


def tiny(seed: int = 1001) -> Workload:
    """1 request, Hq 8 / Hkv 2, 3 of 8 documents x 256 tokens drawn uniformly,
    a 64-token question prefilled causally, then 4 decode steps."""
    wl = build_rag(name="tiny", seed=seed, hq=8, hkv=2, n_docs=8, doc_len=256, docs_per_req=3,
                   alpha=0.0, n_prefill=1, prefill_len=64, prefill_docs_per_req=3)
    # The decode steps continue the same request: its question segment grows
    # from 64 to 68 tokens, one token per step, in the blocks after the chunk.
    st0 = wl.steps[0]
    rng = np.random.default_rng([seed, 4])
    q_first_block = int(wl.store_slot[st0.write_rows[0]]) // BLOCK
    q_off = int(st0.q_pos0[0])
    k = randn_bf16(rng, (4, wl.hkv, wl.d))
    v = randn_bf16(rng, (4, wl.hkv, wl.d))
    n0 = wl.k_store.shape[0]
    wl.k_store = np.concatenate([wl.k_store, k])
    wl.v_store = np.concatenate([wl.v_store, v])
    wl.store_slot = np.concatenate([wl.store_slot,
                                    (q_first_block * BLOCK + 64 + np.arange(4)).astype(np.int32)])
    wl.store_j = np.concatenate([wl.store_j, (64 + np.arange(4)).astype(np.int32)])
    # question tokens 0..63 live at store rows st0.write_rows; 64.. at n0..n0+3,
    # which is not one contiguous store range, so the decode steps describe the
    # question as two oracle segments (same offset, consecutive local indices).
    docs_segs = [(int(st0.seg_src[i]), int(st0.seg_off[i]), int(st0.seg_len[i]))
                 for i in range(st0.seg_indptr[0], st0.seg_indptr[1] - 1)]
    doc_blocks = list(st0.table_block[:st0.table_indptr[1] - _blocks(64)])
    doc_offs = list(st0.table_off[:st0.table_indptr[1] - _blocks(64)])
    for t in range(4):
        n_q = 65 + t
        nb = _blocks(n_q)
        blocks = doc_blocks + list(range(q_first_block, q_first_block + nb))
        offs = doc_offs + [q_off] * nb
        segs = docs_segs + [(int(st0.write_rows[0]), q_off, 64), (n0, q_off + 64, t + 1)]
        gq = np.random.default_rng([seed, 5, t])
        q_raw = randn_bf16(gq, (1, wl.hq, wl.d))
        stp = _make_step("decode", np.array([n0 + t]), q_raw, [[q_off + 64 + t]], [(blocks, offs, segs)])
        wl.steps.append(stp)
    # the pool must hold the 4 extra tokens: 68 tokens -> 5 blocks
    wl.num_blocks = max(wl.num_blocks, q_first_block + _blocks(68))
    return wl


CONFIGS = {
    # name: (constructor kwargs)
    "tiny": None,
    "decode_8b": dict(hq=32, hkv=8, n_docs=1000, doc_len=512, docs_per_req=8, alpha=1.0,
                      n_decode=64, question_len=64),
    "prefill_8b": dict(hq=32, hkv=8, n_docs=1000, doc_len=512, docs_per_req=10, alpha=1.0,
                       n_prefill=16, prefill_len=256),
    # decode 8B with no document shared across requests: 512 of the 1000 documents, each in one request
    "decode_8b_distinct": dict(hq=32, hkv=8, n_docs=1000, doc_len=512, docs_per_req=8, alpha=1.0,
                               n_decode=64, question_len=64, distinct_docs=True),
    "decode_70b": dict(hq=64, hkv=8, n_docs=4000, doc_len=512, docs_per_req=32, alpha=1.2,
                       n_decode=128, question_len=128),
    "decode_70b_uniform": dict(hq=64, hkv=8, n_docs=4000, doc_len=512, docs_per_req=32, alpha=0.0,
                               n_decode=128, question_len=128),
    "mixed_8b": dict(hq=32, hkv=8, n_docs=4000, doc_len=(128, 2048), docs_per_req=8, alpha=1.0,
                     n_prefill=32, prefill_len=256, prefill_docs_per_req=10, n_decode=192,
                     question_len=64, pool_cap_blocks=(1 << 30) // (16 * 8 * 128 * 2 * 2)),
    "mixed_8b_mqa": dict(hq=32, hkv=1, n_docs=4000, doc_len=(128, 2048), docs_per_req=8, alpha=1.0,
                         n_prefill=32, prefill_len=256, prefill_docs_per_req=10, n_decode=192,
                         question_len=64, pool_cap_blocks=(1 << 30) // (16 * 1 * 128 * 2 * 2)),
}

# seeds: 1000 + the configuration's index in the order tiny, decode 8B,
# prefill 8B, decode 70B, mixed 8B
SEEDS = {"tiny": 1001, "decode_8b": 1002, "decode_8b_distinct": 1002, "prefill_8b": 1003, "decode_70b": 1004,
         "decode_70b_uniform": 1004, "mixed_8b": 1005, "mixed_8b_mqa": 1005}


def make(name: str, seed: int | None = None, **overrides) -> Workload:
    """Builds a named workload; overrides change constructor arguments (e.g. alpha, batch sizes)."""
    s = SEEDS[name] if seed is None else seed
    if name == "tiny":
        return tiny(s)
    kw = dict(CONFIGS[name])
    kw.update(overrides)
    return build_rag(name=name, seed=s, **kw)


def with_overrides(step: Step, **kw) -> Step:
    return dataclasses.replace(step, **kw)


# ----------------------------------------------------------------------------- cache-hit streams
def cache_stream(seed: int, n_docs: int = 4000, doc_len=(128, 2048), docs_per_req: int = 8,
                 alpha: float = 1.0, n_requests: int = 20000, order: str = "random"):
    """A seeded stream of RAG requests for cache simulations: per request, docs_per_req distinct
    documents drawn from a finite Zipf(alpha) popularity (rank k has weight k^-alpha), placed in
    random order (order="random") or by popularity rank, most popular first (order="rank", a
    stand-in for ordering by retrieval score).  Returns (doc_tokens [n_docs] int64,
    requests [n_requests][docs_per_req] int64)."""
    if order not in ("random", "rank"):
        raise ValueError(order)
    rng = np.random.default_rng(seed)
    lens = rng.integers(doc_len[0], doc_len[1] + 1, n_docs).astype(np.int64)
    pop = rng.permutation(n_docs)             # document id of popularity rank k
    w = zipf_probs(n_docs, alpha)
    reqs = np.empty((n_requests, docs_per_req), np.int64)
    for r in range(n_requests):
        ranks = rng.choice(n_docs, size=docs_per_req, replace=False, p=w)
        if order == "rank":
            ranks = np.sort(ranks)
        reqs[r] = pop[ranks]
        if order == "random":
            rng.shuffle(reqs[r])
    return lens, reqs
