"""Device-side plumbing around the C ABI: pools, step inputs and launches.

PyTorch only allocates device memory, copies inputs and provides streams;
every step of the hot path runs in liblazy_attn.so through the binding in
``lazy_attn``.  A Workload (from ``workloads``) is turned into:
  * DevicePool -- k_pool, v_pool [num_blocks, Hkv, 16, 128] bf16 and blk_meta
    [num_blocks] uint32 (as int32 storage), filled by lazy_kv_write;
  * DeviceStep -- one step's packed table words, queries, outputs and the
    workspace, with methods that launch the lazy path, the plain path and the
    materialisation of position-adjusted keys.
"""
from __future__ import annotations

import numpy as np
import torch

from . import lazy_attn as la
from .workloads import Step, Workload


def _dev_u16(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)


def _dev_i32(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def cfg_of(wl: Workload) -> la.Cfg:
    return la.Cfg(num_q_heads=wl.hq, num_kv_heads=wl.hkv, rope_base=wl.rope_base)


class DevicePool:
    def __init__(self, wl: Workload, device="cuda", sentinel: int | None = None, cfg: la.Cfg | None = None):
        """cfg: the configuration every call on this pool uses (default: the workload's, RoPE)."""
        self.wl = wl
        self.cfg = cfg_of(wl) if cfg is None else cfg
        self.device = torch.device(device)
        shape = (wl.num_blocks, wl.hkv, 16, wl.d)
        if sentinel is None:
            self.k_pool = torch.zeros(shape, dtype=torch.bfloat16, device=self.device)
            self.v_pool = torch.zeros(shape, dtype=torch.bfloat16, device=self.device)
        else:
            self.k_pool = torch.full(shape, sentinel, dtype=torch.int16, device=self.device).view(torch.bfloat16)
            self.v_pool = torch.full(shape, sentinel, dtype=torch.int16, device=self.device).view(torch.bfloat16)
        self.blk_meta = torch.zeros(wl.num_blocks, dtype=torch.int32, device=self.device)
        self.d_status = torch.zeros(1, dtype=torch.int32, device=self.device)

    def write_rows(self, rows: np.ndarray, chunk: int = 1 << 16, stream=None) -> None:
        """lazy_kv_write of the given token-store rows (documents at setup, new tokens per step)."""
        rows = np.asarray(rows, np.int64)
        for i in range(0, rows.size, chunk):
            r = rows[i:i + chunk]
            if r.size == 0:
                continue
            k = _dev_u16(self.wl.k_store[r], self.device)
            v = _dev_u16(self.wl.v_store[r], self.device)
            slot = _dev_i32(self.wl.store_slot[r], self.device)
            j = _dev_i32(self.wl.store_j[r], self.device)
            la.kv_write(self.cfg, k, v, slot, j, self.k_pool, self.v_pool, self.blk_meta, self.d_status, stream)

    def setup(self) -> "DevicePool":
        self.write_rows(self.wl.setup_rows)
        return self

    def status(self) -> int:
        return int(self.d_status.item())


class DeviceStep:
    """Inputs and outputs of one attention step on the device."""

    def __init__(self, pool: DevicePool, step: Step, with_plain: bool = False):
        self.pool, self.step = pool, step
        dev = pool.device
        wl = pool.wl
        self.cfg = pool.cfg
        self.words_np = la.pack_words(step.table_block, step.table_off)
        self.table = torch.from_numpy(self.words_np.view(np.int32)).to(dev)
        self.table_indptr = _dev_i32(step.table_indptr, dev)
        self.max_words = step.max_words
        self.q_raw = _dev_u16(step.q_raw, dev)
        self.out = torch.zeros((step.total_q, wl.hq, wl.d), dtype=torch.bfloat16, device=dev)
        self.write_rows = step.write_rows
        if step.kind == "decode":
            self.q_pos = _dev_i32(step.q_pos, dev)
            nbytes = la.decode_workspace_bytes(self.cfg, step.num_req, self.max_words)
        else:
            self.cu_q = _dev_i32(step.cu_q, dev)
            self.q_pos0 = _dev_i32(step.q_pos0, dev)
            self.max_q = int(np.diff(step.cu_q).max())
            nbytes = la.prefill_workspace_bytes(self.cfg, step.num_req, step.total_q, self.max_q, self.max_words)
        self.workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
        self.k_mat = None
        if with_plain:
            self.k_mat = torch.empty((self.table.numel(), wl.hkv, 16, wl.d), dtype=torch.bfloat16, device=dev)
            self.out_plain = torch.zeros_like(self.out)

    # ------------------------------------------------------------------ launches
    def write_new_tokens(self, stream=None) -> None:
        self.pool.write_rows(self.write_rows, stream=stream)

    def attend(self, out=None, stream=None) -> None:
        p = self.pool
        out = self.out if out is None else out
        if self.step.kind == "decode":
            la.decode_attn(self.cfg, self.q_raw, self.q_pos, self.table, self.table_indptr, self.max_words,
                           p.blk_meta, p.k_pool, p.v_pool, out, self.workspace, p.d_status, stream)
        else:
            la.prefill_attn(self.cfg, self.q_raw, self.cu_q, self.q_pos0, self.max_q, self.table,
                            self.table_indptr, self.max_words, p.blk_meta, p.k_pool, p.v_pool, out,
                            self.workspace, p.d_status, stream)

    def batch(self) -> dict:
        """This step's arguments as a lazy_mixed_attn batch."""
        b = dict(q_raw=self.q_raw, table=self.table, table_indptr=self.table_indptr, max_words=self.max_words,
                 out=self.out, workspace=self.workspace)
        if self.step.kind == "decode":
            b["q_pos"] = self.q_pos
        else:
            b.update(cu_q=self.cu_q, q_pos0=self.q_pos0, max_q=self.max_q)
        return b

    def materialize(self, stream=None) -> None:
        p = self.pool
        la.materialize_k(self.cfg, self.table, p.blk_meta, p.k_pool, self.k_mat, p.d_status, stream)

    def attend_plain(self, out=None, stream=None) -> None:
        p = self.pool
        out = self.out_plain if out is None else out
        if self.step.kind == "decode":
            la.plain_decode_attn(self.cfg, self.q_raw, self.q_pos, self.table, self.table_indptr, self.max_words,
                                 p.blk_meta, self.k_mat, p.v_pool, out, self.workspace, p.d_status, stream)
        else:
            la.plain_prefill_attn(self.cfg, self.q_raw, self.cu_q, self.q_pos0, self.max_q, self.table,
                                  self.table_indptr, self.max_words, p.blk_meta, self.k_mat, p.v_pool, out,
                                  self.workspace, p.d_status, stream)

    def out_f64(self, out=None) -> np.ndarray:
        o = self.out if out is None else out
        return o.float().cpu().numpy().astype(np.float64).reshape(-1, self.pool.wl.d)


def mixed_attend(prefill: DeviceStep, decode: DeviceStep, stream=None) -> None:
    """One serving step over one pool: the prefill chunks and the decodes in one lazy_mixed_attn call."""
    p = prefill.pool
    assert decode.pool is p, "both batches must use the same pool"
    la.mixed_attn(p.cfg, prefill.batch(), decode.batch(), p.blk_meta, p.k_pool, p.v_pool, p.d_status, stream)

