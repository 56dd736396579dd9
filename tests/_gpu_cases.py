"""Device set-up of hand-shaped cases (tests/_cases.Case) for GPU parity tests.

Each distinct source range of the case's token store becomes one document
stored once in the paged pool (its tokens at local indices 0..len-1); every
segment that uses it becomes table words (block, offset).  Two segments with
the same source therefore share one physical copy, as in the pages' zero-copy
reuse.  By default a document's blocks are consecutive in the pool; with
`scatter_seed` they are placed by a seeded permutation of the pool's blocks, so
that runs of a tile's blocks are (mostly) not consecutive.
"""
from __future__ import annotations

import numpy as np
import torch

from position_agnostic_paged_b200 import lazy_attn as la


def _u16(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)


def _i32(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)


class DeviceCase:
    def __init__(self, case, dev="cuda", extra_blocks: int = 0, scatter_seed: int | None = None,
                 rope_theta=None, alibi_slopes=None):
        self.case = case
        self.cfg = la.Cfg(case.hq, case.hkv, rope_base=case.base,
                          rope_theta=None if rope_theta is None else tuple(float(x) for x in rope_theta),
                          alibi_slopes=None if alibi_slopes is None else tuple(float(x) for x in alibi_slopes))
        docs = {}
        for g in range(case.seg_src.size):
            src, ln = int(case.seg_src[g]), int(case.seg_len[g])
            assert docs.get(src, ln) == ln, "a source must always be used with the same length"
            docs[src] = ln
        self.doc_block = {}
        nb = 0
        for src in sorted(docs):
            self.doc_block[src] = nb
            nb += (docs[src] + 15) // 16
        self.num_blocks = nb + extra_blocks
        # logical block (document-major) -> physical block of the pool
        if scatter_seed is None:
            self.phys = np.arange(max(self.num_blocks, 1))
        else:
            self.phys = np.random.default_rng(scatter_seed).permutation(max(self.num_blocks, 1))
        shape = (max(self.num_blocks, 1), case.hkv, 16, case.d)
        self.k_pool = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
        self.v_pool = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
        self.blk_meta = torch.zeros(shape[0], dtype=torch.int32, device=dev)
        self.d_status = torch.zeros(1, dtype=torch.int32, device=dev)
        rows, slots, js = [], [], []
        for src, ln in docs.items():
            for j in range(ln):
                rows.append(src + j)
                slots.append(int(self.phys[self.doc_block[src] + j // 16]) * 16 + j % 16)
                js.append(j)
        if rows:
            la.kv_write(self.cfg, _u16(case.k_tok[rows], dev), _u16(case.v_tok[rows], dev), _i32(slots, dev),
                        _i32(js, dev), self.k_pool, self.v_pool, self.blk_meta, self.d_status)
        blocks, offs, indptr = [], [], [0]
        for r in range(case.cu_q.size - 1):
            for g in range(case.seg_indptr[r], case.seg_indptr[r + 1]):
                src, off, ln = int(case.seg_src[g]), int(case.seg_off[g]), int(case.seg_len[g])
                for k in range((ln + 15) // 16):
                    blocks.append(int(self.phys[self.doc_block[src] + k]))
                    offs.append(off)
            indptr.append(len(blocks))
        self.words = la.pack_words(np.array(blocks, np.int32), np.array(offs, np.int32))
        self.table = torch.from_numpy(self.words.view(np.int32).copy()).to(dev)
        self.table_indptr = _i32(indptr, dev)
        self.max_words = int(np.diff(indptr).max()) if len(indptr) > 1 else 0
        self.dev = dev

    def decode(self, plain: bool = False):
        c = self.case
        n = c.cu_q.size - 1
        assert np.array_equal(np.diff(c.cu_q), np.ones(n)), "decode: one query per request"
        out = torch.zeros((n, c.hq, c.d), dtype=torch.bfloat16, device=self.dev)
        ws = torch.empty(max(16, la.decode_workspace_bytes(self.cfg, n, self.max_words)), dtype=torch.uint8,
                         device=self.dev)
        q = _u16(c.q_raw, self.dev)
        qp = _i32(c.q_pos, self.dev)
        if plain:
            kmat = torch.empty((self.table.numel(), c.hkv, 16, c.d), dtype=torch.bfloat16, device=self.dev)
            la.materialize_k(self.cfg, self.table, self.blk_meta, self.k_pool, kmat, self.d_status)
            la.plain_decode_attn(self.cfg, q, qp, self.table, self.table_indptr, self.max_words, self.blk_meta,
                                 kmat, self.v_pool, out, ws, self.d_status)
        else:
            la.decode_attn(self.cfg, q, qp, self.table, self.table_indptr, self.max_words, self.blk_meta,
                           self.k_pool, self.v_pool, out, ws, self.d_status)
        return out.float().cpu().numpy().astype(np.float64).reshape(-1, c.d)

    def prefill(self, plain: bool = False, split: bool = True):
        """split: pass the workspace lazy_prefill_workspace_bytes asks for, so that the units of
        a partial last wave run as two halves merged by the combine kernel and the query tiles
        are rotated by the preparation kernel; without it each CTA rotates its own query rows."""
        c = self.case
        n = c.cu_q.size - 1
        q_pos0 = []
        for r in range(n):
            qp = c.q_pos[c.cu_q[r]:c.cu_q[r + 1]]
            assert qp.size == 0 or np.array_equal(qp, qp[0] + np.arange(qp.size)), \
                "prefill: contiguous query positions"
            q_pos0.append(int(qp[0]) if qp.size else 0)
        total_q = int(c.cu_q[-1])
        max_q = int(np.diff(c.cu_q).max())
        out = torch.zeros((total_q, c.hq, c.d), dtype=torch.bfloat16, device=self.dev)
        q = _u16(c.q_raw, self.dev)
        cu = _i32(c.cu_q, self.dev)
        p0 = _i32(q_pos0, self.dev)
        ws = None
        if split:
            nb = la.prefill_workspace_bytes(self.cfg, n, total_q, max_q, self.max_words)
            ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=self.dev)
        if plain:
            kmat = torch.empty((self.table.numel(), c.hkv, 16, c.d), dtype=torch.bfloat16, device=self.dev)
            la.materialize_k(self.cfg, self.table, self.blk_meta, self.k_pool, kmat, self.d_status)
            la.plain_prefill_attn(self.cfg, q, cu, p0, max_q, self.table, self.table_indptr, self.max_words,
                                  self.blk_meta, kmat, self.v_pool, out, ws, self.d_status)
        else:
            la.prefill_attn(self.cfg, q, cu, p0, max_q, self.table, self.table_indptr, self.max_words,
                            self.blk_meta, self.k_pool, self.v_pool, out, ws, self.d_status)
        return out.float().cpu().numpy().astype(np.float64).reshape(-1, c.d)

    def mixed_batches(self, n_prefill: int):
        """Requests 0..n_prefill-1 as a prefill batch (contiguous query positions), the rest as a
        decode batch (one query each), both over this case's pool and table (the batches index the
        one table through slices of its row pointer)."""
        c = self.case
        n = c.cu_q.size - 1
        cu = c.cu_q
        tp = int(cu[n_prefill])
        assert np.array_equal(np.diff(cu[n_prefill:]), np.ones(n - n_prefill)), "decode: one query per request"
        pf_cu = cu[: n_prefill + 1]
        q_pos0 = [int(c.q_pos[cu[r]]) if cu[r + 1] > cu[r] else 0 for r in range(n_prefill)]
        max_q = int(np.diff(pf_cu).max())
        pf = dict(q_raw=_u16(c.q_raw[:tp], self.dev), cu_q=_i32(pf_cu, self.dev), q_pos0=_i32(q_pos0, self.dev),
                  max_q=max_q, table=self.table, table_indptr=self.table_indptr[: n_prefill + 1],
                  max_words=self.max_words,
                  out=torch.zeros((tp, c.hq, c.d), dtype=torch.bfloat16, device=self.dev),
                  workspace=torch.empty(max(16, la.prefill_workspace_bytes(self.cfg, n_prefill, tp, max_q,
                                                                           self.max_words)),
                                        dtype=torch.uint8, device=self.dev))
        nd = n - n_prefill
        dc = dict(q_raw=_u16(c.q_raw[tp:], self.dev), q_pos=_i32(c.q_pos[tp:], self.dev), table=self.table,
                  table_indptr=self.table_indptr[n_prefill:], max_words=self.max_words,
                  out=torch.zeros((nd, c.hq, c.d), dtype=torch.bfloat16, device=self.dev),
                  workspace=torch.empty(max(16, la.decode_workspace_bytes(self.cfg, nd, self.max_words)),
                                        dtype=torch.uint8, device=self.dev))
        return pf, dc

    def mixed(self, pf, dc, stream=None):
        la.mixed_attn(self.cfg, pf, dc, self.blk_meta, self.k_pool, self.v_pool, self.d_status, stream)

    def separate(self, pf, dc):
        la.prefill_attn(self.cfg, pf["q_raw"], pf["cu_q"], pf["q_pos0"], pf["max_q"], pf["table"],
                        pf["table_indptr"], pf["max_words"], self.blk_meta, self.k_pool, self.v_pool, pf["out"],
                        pf["workspace"], self.d_status)
        la.decode_attn(self.cfg, dc["q_raw"], dc["q_pos"], dc["table"], dc["table_indptr"], dc["max_words"],
                       self.blk_meta, self.k_pool, self.v_pool, dc["out"], dc["workspace"], self.d_status)

    def status(self) -> int:
        return int(self.d_status.item())
