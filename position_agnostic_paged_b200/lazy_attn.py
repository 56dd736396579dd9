"""Thin ctypes binding of liblazy_attn.so (include/lazy_attn.h).

Argument marshalling only: every function takes torch tensors that already
live on the GPU, passes their data pointers and the current CUDA stream to the
C entry point of the same name, and raises LazyAttnError on a non-zero return
code.  All computation happens in the library's CUDA kernels; there is no CPU
fallback, and importing this module fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblazy_attn.so")

LAZY_OK, LAZY_EINVAL, LAZY_ERANGE, LAZY_ESHAPE, LAZY_EWORKSPACE, LAZY_ECUDA = 0, -1, -2, -3, -4, -5
DSTATUS_BAD_BLOCK, DSTATUS_BAD_SLOT, DSTATUS_BAD_ALIGN, DSTATUS_BAD_TABLE, DSTATUS_TIMEOUT = 1, 2, 4, 8, 16

EXPORTED = [
    "lazy_version", "lazy_strerror", "lazy_pack_words", "lazy_kv_write",
    "lazy_decode_workspace_bytes", "lazy_decode_attn",
    "lazy_prefill_workspace_bytes", "lazy_prefill_attn",
    "lazy_materialize_k", "lazy_plain_decode_attn", "lazy_plain_prefill_attn",
    "lazy_debug_decode_table", "lazy_decode_attn_noalloc", "lazy_decode_noalloc_capacity",
    "lazy_cache_create", "lazy_cache_destroy", "lazy_cache_access", "lazy_cache_contains", "lazy_cache_stats",
    "lazy_mixed_attn", "lazy_rope_theta", "lazy_rope_theta_llama31", "lazy_alibi_slopes",
    "lazy_debug_bounded_wait",
]


class LazyAttnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {code}: {strerror(code)}")
        self.code = code


class LazyAttnCfg(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("block_size", ctypes.c_int), ("rope_base", ctypes.c_float), ("softmax_scale", ctypes.c_float),
                ("rope_theta", ctypes.POINTER(ctypes.c_double)),
                ("alibi_slopes", ctypes.POINTER(ctypes.c_double))]


@dataclass(frozen=True)
class Cfg:
    """rope_theta: optional head_dim/2 RoPE frequencies (e.g. rope.llama31_theta()) in place of
    rope_base^(-2i/head_dim).  alibi_slopes: optional num_q_heads ALiBi slopes (e.g.
    rope.alibi_slopes(num_q_heads)) in place of RoPE: keys are stored as given and each score gets
    -slope_h * (query position - key position)."""
    num_q_heads: int
    num_kv_heads: int
    rope_base: float = 500000.0
    head_dim: int = 128
    block_size: int = 16
    softmax_scale: float = 0.0
    rope_theta: tuple | None = None
    alibi_slopes: tuple | None = None

    def c(self) -> LazyAttnCfg:
        st = LazyAttnCfg(self.num_q_heads, self.num_kv_heads, self.head_dim, self.block_size,
                         float(self.rope_base), float(self.softmax_scale), None, None)
        if self.alibi_slopes is not None:
            if len(self.alibi_slopes) != self.num_q_heads:
                raise ValueError("alibi_slopes needs one slope per query head")
            sl = (ctypes.c_double * len(self.alibi_slopes))(*[float(x) for x in self.alibi_slopes])
            st._alibi_keepalive = sl
            st.alibi_slopes = ctypes.cast(sl, ctypes.POINTER(ctypes.c_double))
        if self.rope_theta is not None:
            arr = (ctypes.c_double * len(self.rope_theta))(*[float(x) for x in self.rope_theta])
            st._theta_keepalive = arr
            st.rope_theta = ctypes.cast(arr, ctypes.POINTER(ctypes.c_double))
        return st


_vp, _i, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_cfgp = ctypes.POINTER(LazyAttnCfg)


class PrefillBatch(ctypes.Structure):
    """lazy_prefill_batch: the arguments of lazy_prefill_attn for one batch."""
    _fields_ = [("q_raw", _vp), ("cu_q", _vp), ("q_pos0", _vp), ("num_req", _i), ("total_q", _i), ("max_q", _i),
                ("table", _vp), ("table_indptr", _vp), ("max_words", _i), ("out", _vp), ("workspace", _vp),
                ("ws_bytes", _sz)]


class DecodeBatch(ctypes.Structure):
    """lazy_decode_batch: the arguments of lazy_decode_attn for one batch."""
    _fields_ = [("q_raw", _vp), ("q_pos", _vp), ("num_req", _i), ("table", _vp), ("table_indptr", _vp),
                ("max_words", _i), ("out", _vp), ("workspace", _vp), ("ws_bytes", _sz)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m position_agnostic_paged_b200.build` "
                          "(the CUDA library is required; there is no fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "lazy_version": (_i, []),
        "lazy_strerror": (ctypes.c_char_p, [_i]),
        "lazy_pack_words": (_i, [_vp, _vp, _i64, _vp]),
        "lazy_kv_write": (_i, [_cfgp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp]),
        "lazy_decode_workspace_bytes": (_sz, [_cfgp, _i, _i]),
        "lazy_decode_attn": (_i, [_cfgp, _vp, _vp, _i, _vp, _vp, _i, _vp, _vp, _vp, _i, _vp, _vp, _sz, _vp, _vp]),
        "lazy_prefill_workspace_bytes": (_sz, [_cfgp, _i, _i, _i, _i]),
        "lazy_prefill_attn": (_i, [_cfgp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _i, _vp, _vp, _vp, _i, _vp, _vp,
                                   _sz, _vp, _vp]),
        "lazy_materialize_k": (_i, [_cfgp, _vp, _i, _vp, _vp, _i, _vp, _vp, _vp]),
        "lazy_plain_decode_attn": (_i, [_cfgp, _vp, _vp, _i, _vp, _vp, _i, _vp, _vp, _i, _vp, _i, _vp, _vp, _sz,
                                        _vp, _vp]),
        "lazy_plain_prefill_attn": (_i, [_cfgp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _i, _vp, _vp, _i, _vp, _i,
                                         _vp, _vp, _sz, _vp, _vp]),
        "lazy_debug_decode_table": (_i, [_vp, _i64, _vp, _i, _vp, _vp, _vp, _vp, _vp]),
        "lazy_decode_attn_noalloc": (_i, [_cfgp, _vp, _vp, _i, _vp, _vp, _i, _vp, _vp, _vp, _i, _vp, _vp, _vp]),
        "lazy_decode_noalloc_capacity": (_sz, []),
        "lazy_mixed_attn": (_i, [_cfgp, ctypes.POINTER(PrefillBatch), ctypes.POINTER(DecodeBatch), _vp, _vp, _vp, _i,
                                 _vp, _vp]),
        "lazy_rope_theta": (_i, [ctypes.c_double, _i, _vp]),
        "lazy_rope_theta_llama31": (_i, [ctypes.c_double, _i, ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                         ctypes.c_double, _vp]),
        "lazy_alibi_slopes": (_i, [_i, _vp]),
        "lazy_debug_bounded_wait": (_i, [ctypes.c_uint32, _i, _vp, _vp, _vp]),
        "lazy_cache_create": (_vp, [_i64]),
        "lazy_cache_destroy": (None, [_vp]),
        "lazy_cache_access": (_i, [_vp, ctypes.c_uint64, ctypes.c_int32, _vp]),
        "lazy_cache_contains": (_i, [_vp, ctypes.c_uint64]),
        "lazy_cache_stats": (_i, [_vp, _vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def version() -> int:
    return int(_lib.lazy_version())


def strerror(code: int) -> str:
    return _lib.lazy_strerror(int(code)).decode()


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise LazyAttnError(fn, rc)


def _ptr(t) -> int | None:
    if t is None:
        return None
    return int(t.data_ptr())


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream) or None
    return int(getattr(stream, "cuda_stream", stream)) or None


def pack_words(block: np.ndarray, offset: np.ndarray) -> np.ndarray:
    """Host codec: (block, offset) int32 arrays -> uint32 table words (raises on overflow)."""
    block = np.ascontiguousarray(block, np.int32)
    offset = np.ascontiguousarray(offset, np.int32)
    out = np.empty(block.size, np.uint32)
    _check("lazy_pack_words", _lib.lazy_pack_words(block.ctypes.data, offset.ctypes.data, block.size,
                                                   out.ctypes.data))
    return out


def rope_theta(base: float, head_dim: int) -> tuple[float, ...]:
    """lazy_rope_theta: theta_i = base^(-2i/head_dim)."""
    out = np.empty(max(int(head_dim) // 2, 1), np.float64)
    _check("lazy_rope_theta", _lib.lazy_rope_theta(float(base), int(head_dim), out.ctypes.data))
    return tuple(float(x) for x in out[: int(head_dim) // 2])


def rope_theta_llama31(base: float, head_dim: int, factor: float, low_freq_factor: float,
                       high_freq_factor: float, original_max_position: float) -> tuple[float, ...]:
    """lazy_rope_theta_llama31: frequencies with Llama-3.1 scaling."""
    out = np.empty(max(int(head_dim) // 2, 1), np.float64)
    _check("lazy_rope_theta_llama31", _lib.lazy_rope_theta_llama31(
        float(base), int(head_dim), float(factor), float(low_freq_factor), float(high_freq_factor),
        float(original_max_position), out.ctypes.data))
    return tuple(float(x) for x in out[: int(head_dim) // 2])


def alibi_slopes(num_heads: int) -> tuple[float, ...]:
    """lazy_alibi_slopes: the ALiBi paper's head slopes."""
    out = np.empty(max(int(num_heads), 1), np.float64)
    _check("lazy_alibi_slopes", _lib.lazy_alibi_slopes(int(num_heads), out.ctypes.data))
    return tuple(float(x) for x in out[: int(num_heads)])


def kv_write(cfg: Cfg, k_raw, v_raw, slot, local_j, k_pool, v_pool, blk_meta, d_status=None, stream=None):
    c = cfg.c()
    _check("lazy_kv_write", _lib.lazy_kv_write(
        ctypes.byref(c), _ptr(k_raw), _ptr(v_raw), int(slot.numel()), _ptr(slot), _ptr(local_j),
        _ptr(k_pool), _ptr(v_pool), _ptr(blk_meta), int(k_pool.shape[0]), _ptr(d_status), _stream(stream)))


def decode_workspace_bytes(cfg: Cfg, num_req: int, max_words: int) -> int:
    c = cfg.c()
    return int(_lib.lazy_decode_workspace_bytes(ctypes.byref(c), int(num_req), int(max_words)))


def prefill_workspace_bytes(cfg: Cfg, num_req: int, total_q: int, max_q: int, max_words: int) -> int:
    c = cfg.c()
    return int(_lib.lazy_prefill_workspace_bytes(ctypes.byref(c), int(num_req), int(total_q), int(max_q),
                                                 int(max_words)))


def decode_attn(cfg: Cfg, q_raw, q_pos, table, table_indptr, max_words: int, blk_meta, k_pool, v_pool, out,
                workspace, d_status=None, stream=None):
    c = cfg.c()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("lazy_decode_attn", _lib.lazy_decode_attn(
        ctypes.byref(c), _ptr(q_raw), _ptr(q_pos), int(q_pos.numel()), _ptr(table), _ptr(table_indptr),
        int(max_words), _ptr(blk_meta), _ptr(k_pool), _ptr(v_pool), int(k_pool.shape[0]), _ptr(out),
        _ptr(workspace), ws_bytes, _ptr(d_status), _stream(stream)))


def prefill_attn(cfg: Cfg, q_raw, cu_q, q_pos0, max_q: int, table, table_indptr, max_words: int, blk_meta,
                 k_pool, v_pool, out, workspace=None, d_status=None, stream=None):
    c = cfg.c()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("lazy_prefill_attn", _lib.lazy_prefill_attn(
        ctypes.byref(c), _ptr(q_raw), _ptr(cu_q), _ptr(q_pos0), int(q_pos0.numel()), int(q_raw.shape[0]),
        int(max_q), _ptr(table), _ptr(table_indptr), int(max_words), _ptr(blk_meta), _ptr(k_pool),
        _ptr(v_pool), int(k_pool.shape[0]), _ptr(out), _ptr(workspace), ws_bytes, _ptr(d_status),
        _stream(stream)))


def _nbytes(t) -> int:
    return t.numel() * t.element_size() if t is not None else 0


def mixed_attn(cfg: Cfg, prefill: dict | None, decode: dict | None, blk_meta, k_pool, v_pool, d_status=None,
               stream=None):
    """One serving step with prefill chunks and decodes (lazy_mixed_attn): the results of
    prefill_attn(**prefill) and decode_attn(**decode), both batches validated before either runs,
    then run in that order on `stream`.

    prefill: dict(q_raw, cu_q, q_pos0, max_q, table, table_indptr, max_words, out, workspace);
    decode: dict(q_raw, q_pos, table, table_indptr, max_words, out, workspace).  The two
    workspaces must be distinct."""
    c = cfg.c()
    pf = dc = None
    if prefill is not None:
        b = prefill
        pf = PrefillBatch(_ptr(b["q_raw"]), _ptr(b["cu_q"]), _ptr(b["q_pos0"]), int(b["q_pos0"].numel()),
                          int(b["q_raw"].shape[0]), int(b["max_q"]), _ptr(b["table"]), _ptr(b["table_indptr"]),
                          int(b["max_words"]), _ptr(b["out"]), _ptr(b.get("workspace")), _nbytes(b.get("workspace")))
    if decode is not None:
        b = decode
        dc = DecodeBatch(_ptr(b["q_raw"]), _ptr(b["q_pos"]), int(b["q_pos"].numel()), _ptr(b["table"]),
                         _ptr(b["table_indptr"]), int(b["max_words"]), _ptr(b["out"]), _ptr(b["workspace"]),
                         _nbytes(b["workspace"]))
    _check("lazy_mixed_attn", _lib.lazy_mixed_attn(
        ctypes.byref(c), ctypes.byref(pf) if pf is not None else None, ctypes.byref(dc) if dc is not None else None,
        _ptr(blk_meta), _ptr(k_pool), _ptr(v_pool), int(k_pool.shape[0]), _ptr(d_status), _stream(stream)))


def materialize_k(cfg: Cfg, table, blk_meta, k_pool, k_mat, d_status=None, stream=None):
    c = cfg.c()
    _check("lazy_materialize_k", _lib.lazy_materialize_k(
        ctypes.byref(c), _ptr(table), int(table.numel()), _ptr(blk_meta), _ptr(k_pool), int(k_pool.shape[0]),
        _ptr(k_mat), _ptr(d_status), _stream(stream)))


def plain_decode_attn(cfg: Cfg, q_raw, q_pos, table, table_indptr, max_words: int, blk_meta, k_mat, v_pool, out,
                      workspace, d_status=None, stream=None):
    c = cfg.c()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("lazy_plain_decode_attn", _lib.lazy_plain_decode_attn(
        ctypes.byref(c), _ptr(q_raw), _ptr(q_pos), int(q_pos.numel()), _ptr(table), _ptr(table_indptr),
        int(max_words), _ptr(blk_meta), _ptr(k_mat), int(k_mat.shape[0]), _ptr(v_pool), int(v_pool.shape[0]),
        _ptr(out), _ptr(workspace), ws_bytes, _ptr(d_status), _stream(stream)))


def plain_prefill_attn(cfg: Cfg, q_raw, cu_q, q_pos0, max_q: int, table, table_indptr, max_words: int, blk_meta,
                       k_mat, v_pool, out, workspace=None, d_status=None, stream=None):
    c = cfg.c()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("lazy_plain_prefill_attn", _lib.lazy_plain_prefill_attn(
        ctypes.byref(c), _ptr(q_raw), _ptr(cu_q), _ptr(q_pos0), int(q_pos0.numel()), int(q_raw.shape[0]),
        int(max_q), _ptr(table), _ptr(table_indptr), int(max_words), _ptr(blk_meta), _ptr(k_mat),
        int(k_mat.shape[0]), _ptr(v_pool), int(v_pool.shape[0]), _ptr(out), _ptr(workspace), ws_bytes,
        _ptr(d_status), _stream(stream)))


def debug_decode_table(table, blk_meta, num_blocks: int, out_block, out_slot, out_pos, d_status=None, stream=None):
    _check("lazy_debug_decode_table", _lib.lazy_debug_decode_table(
        _ptr(table), int(table.numel()), _ptr(blk_meta), int(num_blocks), _ptr(out_block), _ptr(out_slot),
        _ptr(out_pos), _ptr(d_status), _stream(stream)))


def debug_bounded_wait(polls: int, complete: bool, result, d_status=None, stream=None):
    """lazy_debug_bounded_wait: a bounded mbarrier wait that runs out (complete=False) or succeeds."""
    _check("lazy_debug_bounded_wait", _lib.lazy_debug_bounded_wait(
        int(polls), 1 if complete else 0, _ptr(result), _ptr(d_status), _stream(stream)))


def decode_noalloc_capacity() -> int:
    """Bytes of the library's built-in scratch array used by decode_attn_noalloc."""
    return int(_lib.lazy_decode_noalloc_capacity())


def decode_attn_noalloc(cfg: Cfg, q_raw, q_pos, table, table_indptr, max_words: int, blk_meta, k_pool, v_pool, out,
                        d_status=None, stream=None):
    """decode_attn without a workspace, for callers that cannot allocate device memory.

    The split partials live in a fixed array inside the library (see
    decode_noalloc_capacity()); calls that may overlap on the GPU must be
    serialised by the caller.  Raises LazyAttnError(LAZY_ERANGE) when the
    batch needs more scratch than the array holds.
    """
    c = cfg.c()
    _check("lazy_decode_attn_noalloc", _lib.lazy_decode_attn_noalloc(
        ctypes.byref(c), _ptr(q_raw), _ptr(q_pos), int(q_pos.numel()), _ptr(table), _ptr(table_indptr),
        int(max_words), _ptr(blk_meta), _ptr(k_pool), _ptr(v_pool), int(k_pool.shape[0]), _ptr(out),
        _ptr(d_status), _stream(stream)))


class BlockCache:
    """Host-side LRU cache of pool blocks (lazy_cache_*): key -> the blocks of one cached entry.

    access(key, n_blocks) returns (hit, block_ids); on a miss the blocks are freshly allocated
    (after evicting least recently used entries) and the caller writes the entry there.  An entry
    larger than the cache is counted as a miss and returns (False, None).
    """

    STAT_NAMES = ("hits", "misses", "hit_blocks", "miss_blocks", "evictions", "used_blocks", "entries",
                  "free_extents")

    def __init__(self, capacity_blocks: int):
        self._h = _lib.lazy_cache_create(int(capacity_blocks))
        if not self._h:
            raise LazyAttnError("lazy_cache_create", LAZY_EINVAL)
        self.capacity = int(capacity_blocks)
        self._buf = (ctypes.c_int32 * 1)()

    def close(self) -> None:
        if self._h:
            _lib.lazy_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def access(self, key: int, n_blocks: int):
        if len(self._buf) < n_blocks:
            self._buf = (ctypes.c_int32 * max(n_blocks, 2 * len(self._buf)))()
        rc = _lib.lazy_cache_access(self._h, ctypes.c_uint64(int(key) & 0xFFFFFFFFFFFFFFFF), int(n_blocks),
                                    ctypes.cast(self._buf, ctypes.c_void_p))
        if rc == LAZY_ERANGE:
            return False, None
        if rc < 0:
            raise LazyAttnError("lazy_cache_access", rc)
        return rc == 1, np.frombuffer(self._buf, dtype=np.int32, count=n_blocks).copy()

    def contains(self, key: int) -> bool:
        return _lib.lazy_cache_contains(self._h, ctypes.c_uint64(int(key) & 0xFFFFFFFFFFFFFFFF)) == 1

    def stats(self) -> dict:
        out = (ctypes.c_int64 * 8)()
        _check("lazy_cache_stats", _lib.lazy_cache_stats(self._h, ctypes.cast(out, ctypes.c_void_p)))
        return dict(zip(self.STAT_NAMES, [int(x) for x in out]))
