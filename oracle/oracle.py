"""ctypes wrapper around ``lazy_oracle.c`` (TEST INFRASTRUCTURE ONLY).

Every function below marshals numpy arrays into the C oracle and back; the
arithmetic itself is in the C file, which cites the pages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lazy_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD_DIR, "liblazy_oracle.so")
_lock = threading.Lock()
_lib = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f64p = ctypes.POINTER(ctypes.c_double)


def lib_path() -> str:
    return _LIB


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP on) unless an up-to-date build exists."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=gnu99", "-fopenmp", "-fPIC", "-shared", "-Wall",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def load_library(path: str):
    """Loads a compiled oracle from path and declares its C signatures."""
    lib = ctypes.CDLL(path)
    _bind(lib)
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(build())
    return _lib


def _bind(lib) -> None:
    lib.oracle_bf16_to_f64.restype = ctypes.c_double
    lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
    lib.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
    lib.oracle_pack_word.restype = ctypes.c_int
    lib.oracle_pack_word.argtypes = [ctypes.c_int64, ctypes.c_int64, _u32p]
    lib.oracle_unpack_word.restype = None
    lib.oracle_unpack_word.argtypes = [ctypes.c_uint32, _i32p, _i32p]
    lib.oracle_pack_meta.restype = ctypes.c_uint32
    lib.oracle_pack_meta.argtypes = [ctypes.c_int32, ctypes.c_int32]
    lib.oracle_rope.restype = None
    lib.oracle_rope.argtypes = [_f64p, ctypes.c_int, ctypes.c_double, ctypes.c_int64, _f64p]
    lib.oracle_kv_write.restype = ctypes.c_int
    lib.oracle_kv_write.argtypes = [
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
        _u16p, _u16p, _i32p, _i32p, ctypes.c_int64, _u16p, _u16p, _u32p]
    lib.oracle_expand_table.restype = ctypes.c_int
    lib.oracle_expand_table.argtypes = [
        ctypes.c_int64, _u32p, _u32p, ctypes.c_int64, _i32p, _i32p, _i32p]
    lib.oracle_attend.restype = ctypes.c_int
    lib.oracle_attend.argtypes = [
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_double, ctypes.c_double,
        _u16p, _i32p, _i32p,
        _i32p, _i32p, _i32p, _i32p,
        _u16p, _u16p,
        ctypes.c_int64, _i32p, _i32p,
        _f64p, _f64p, ctypes.c_int64]
    lib.oracle_rope_rows_bf16.restype = ctypes.c_int
    lib.oracle_rope_rows_bf16.argtypes = [
        ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_double, _u16p, _i32p, _u16p]
    lib.oracle_set_rope_theta.restype = None
    lib.oracle_set_rope_theta.argtypes = [_f64p, ctypes.c_int]
    lib.oracle_set_alibi.restype = None
    lib.oracle_set_alibi.argtypes = [_f64p, ctypes.c_int]
    lib.oracle_alibi_slopes.restype = None
    lib.oracle_alibi_slopes.argtypes = [ctypes.c_int, _f64p]
    lib.oracle_llama31_theta.restype = None
    lib.oracle_llama31_theta.argtypes = [ctypes.c_double, ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                         ctypes.c_double, ctypes.c_double, _f64p]
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_set_num_threads.restype = None
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]


def _p(a: np.ndarray, ct):
    return a.ctypes.data_as(ct)


class _Theta:
    """Sets the oracle's RoPE frequency table for one call (None: base^(-2i/d))."""

    def __init__(self, lib, theta):
        self.lib = lib
        self.theta = None if theta is None else _c(theta, np.float64)

    def __enter__(self):
        if self.theta is not None:
            self.lib.oracle_set_rope_theta(_p(self.theta, _f64p), int(self.theta.size))
        return self

    def __exit__(self, *exc):
        if self.theta is not None:
            self.lib.oracle_set_rope_theta(ctypes.cast(None, _f64p), 0)
        return False


class _Alibi:
    """Sets the oracle's ALiBi slopes (one per query head) for one call (None: RoPE)."""

    def __init__(self, lib, slopes):
        self.lib = lib
        self.slopes = None if slopes is None else _c(slopes, np.float64)

    def __enter__(self):
        if self.slopes is not None:
            self.lib.oracle_set_alibi(_p(self.slopes, _f64p), int(self.slopes.size))
        return self

    def __exit__(self, *exc):
        if self.slopes is not None:
            self.lib.oracle_set_alibi(ctypes.cast(None, _f64p), 0)
        return False


def alibi_slopes(n_heads: int, lib=None) -> np.ndarray:
    """The ALiBi paper's head slopes for n_heads heads (the oracle's own computation)."""
    out = np.empty(n_heads, np.float64)
    (lib or _load()).oracle_alibi_slopes(int(n_heads), _p(out, _f64p))
    return out


def llama31_theta(base: float = 500000.0, d: int = 128, factor: float = 8.0, low_factor: float = 1.0,
                  high_factor: float = 4.0, original_max: float = 8192.0) -> np.ndarray:
    """RoPE frequencies with Llama-3.1 frequency scaling (the oracle's own computation)."""
    out = np.empty(d // 2, np.float64)
    _load().oracle_llama31_theta(float(base), int(d), float(factor), float(low_factor), float(high_factor),
                                 float(original_max), _p(out, _f64p))
    return out


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def bf16_to_f64(bits) -> np.ndarray:
    lib = _load()
    b = _c(bits, np.uint16).ravel()
    return np.array([lib.oracle_bf16_to_f64(int(x)) for x in b], dtype=np.float64).reshape(np.shape(bits))


def f64_to_bf16(x) -> np.ndarray:
    lib = _load()
    a = _c(x, np.float64).ravel()
    return np.array([lib.oracle_f64_to_bf16(float(v)) for v in a], dtype=np.uint16).reshape(np.shape(x))


def pack_word(block: int, offset: int) -> int:
    """Returns the packed word, or raises ValueError when a field overflows."""
    w = ctypes.c_uint32(0)
    rc = _load().oracle_pack_word(int(block), int(offset), ctypes.byref(w))
    if rc != 0:
        raise ValueError(f"table word field out of range: block={block} offset={offset}")
    return int(w.value)


def unpack_word(word: int) -> tuple[int, int]:
    b, o = ctypes.c_int32(0), ctypes.c_int32(0)
    _load().oracle_unpack_word(int(word), ctypes.byref(b), ctypes.byref(o))
    return int(b.value), int(o.value)


def pack_meta(block_index_in_segment: int, n_valid: int) -> int:
    return int(_load().oracle_pack_meta(int(block_index_in_segment), int(n_valid)))


def rope(x, pos: int, base: float, theta=None) -> np.ndarray:
    x = _c(x, np.float64)
    y = np.empty_like(x)
    lib = _load()
    with _Theta(lib, theta):
        lib.oracle_rope(_p(x, _f64p), int(x.shape[-1]), float(base), int(pos), _p(y, _f64p))
    return y


def kv_write(k_raw, v_raw, slot, local_j, k_pool, v_pool, blk_meta, base: float, theta=None) -> int:
    """Applies the expected effect of a pool write in place on numpy arrays.

    k_raw, v_raw: uint16 [n_tok, Hkv, d]; k_pool, v_pool: uint16 [nb, Hkv, 16, d];
    blk_meta: uint32 [nb].  Returns the oracle's status code.
    """
    k_raw = _c(k_raw, np.uint16)
    v_raw = _c(v_raw, np.uint16)
    slot = _c(slot, np.int32)
    local_j = _c(local_j, np.int32)
    assert k_pool.flags.c_contiguous and v_pool.flags.c_contiguous and blk_meta.flags.c_contiguous
    assert k_pool.dtype == np.uint16 and v_pool.dtype == np.uint16 and blk_meta.dtype == np.uint32
    n_tok, hkv, d = k_raw.shape
    lib = _load()
    with _Theta(lib, theta):
        return int(lib.oracle_kv_write(
            int(n_tok), int(hkv), int(d), float(base), _p(k_raw, _u16p), _p(v_raw, _u16p),
            _p(slot, _i32p), _p(local_j, _i32p), int(k_pool.shape[0]),
            _p(k_pool, _u16p), _p(v_pool, _u16p), _p(blk_meta, _u32p)))


def expand_table(words, blk_meta, num_blocks: int):
    """Returns (block, slot, pos) int32 arrays of shape [n_words, 16] and the status."""
    words = _c(words, np.uint32).ravel()
    blk_meta = _c(blk_meta, np.uint32)
    n = words.size
    ob = np.empty((n, 16), np.int32)
    osl = np.empty((n, 16), np.int32)
    op = np.empty((n, 16), np.int32)
    rc = _load().oracle_expand_table(int(n), _p(words, _u32p), _p(blk_meta, _u32p), int(num_blocks),
                                     _p(ob, _i32p), _p(osl, _i32p), _p(op, _i32p))
    return ob, osl, op, int(rc)


def attend(*, num_q_heads: int, num_kv_heads: int, rope_base: float, q_raw, cu_q, q_pos,
           seg_indptr, seg_src, seg_off, seg_len, k_tok, v_tok, sel_q=None, sel_h=None,
           softmax_scale: float = 0.0, want_scores: bool = False, lib=None, rope_theta=None,
           alibi_slopes=None):
    """Materialised causal GQA attention in fp64.

    q_raw: uint16 [total_q, Hq, d]; k_tok, v_tok: uint16 [n_store, Hkv, d].
    Returns out [n_rows, d] float64 (rows: the selection, or every (q, h) in
    q-major order) and, if want_scores, scores [n_rows, max_kv_len].
    alibi_slopes (one per query head) replaces RoPE by the linear ALiBi penalty.
    """
    q_raw = _c(q_raw, np.uint16)
    k_tok = _c(k_tok, np.uint16)
    v_tok = _c(v_tok, np.uint16)
    cu_q = _c(cu_q, np.int32)
    q_pos = _c(q_pos, np.int32)
    seg_indptr = _c(seg_indptr, np.int32)
    seg_src = _c(seg_src, np.int32)
    seg_off = _c(seg_off, np.int32)
    seg_len = _c(seg_len, np.int32)
    num_req = cu_q.size - 1
    d = q_raw.shape[-1]
    total_q = int(cu_q[-1])
    if sel_q is None:
        n_sel = -1
        n_rows = total_q * num_q_heads
        sq = np.zeros(1, np.int32)
        sh = np.zeros(1, np.int32)
    else:
        sq = _c(sel_q, np.int32)
        sh = _c(sel_h, np.int32)
        n_sel = n_rows = sq.size
    out = np.zeros((max(n_rows, 1), d), np.float64)
    if want_scores:
        kv_lens = [int(seg_len[seg_indptr[r]:seg_indptr[r + 1]].sum()) for r in range(num_req)]
        ld = max(kv_lens + [1])
        scores = np.full((max(n_rows, 1), ld), np.nan, np.float64)
        sp = _p(scores, _f64p)
    else:
        ld = 0
        scores = None
        sp = ctypes.cast(None, _f64p)
    lib = lib or _load()
    if alibi_slopes is not None and len(alibi_slopes) != num_q_heads:
        raise ValueError("alibi_slopes needs one slope per query head")
    with _Theta(lib, rope_theta), _Alibi(lib, alibi_slopes):
        rc = lib.oracle_attend(
            int(num_req), int(num_q_heads), int(num_kv_heads), int(d), float(rope_base),
            float(softmax_scale), _p(q_raw, _u16p), _p(cu_q, _i32p), _p(q_pos, _i32p),
            _p(seg_indptr, _i32p), _p(seg_src, _i32p), _p(seg_off, _i32p), _p(seg_len, _i32p),
            _p(k_tok, _u16p), _p(v_tok, _u16p), int(n_sel), _p(sq, _i32p), _p(sh, _i32p),
            _p(out, _f64p), sp, int(ld))
    if rc != 0:
        raise RuntimeError(f"oracle_attend failed with status {rc}")
    out = out[:n_rows]
    if want_scores:
        return out, scores[:n_rows]
    return out


def rope_rows_bf16(k_raw, pos, base: float, theta=None) -> np.ndarray:
    """bf16(RoPE(k_raw[n], pos[n])) for uint16 k_raw [n, Hkv, d]."""
    k_raw = _c(k_raw, np.uint16)
    pos = _c(pos, np.int32)
    out = np.empty_like(k_raw)
    n, hkv, d = k_raw.shape
    lib = _load()
    with _Theta(lib, theta):
        rc = lib.oracle_rope_rows_bf16(int(n), int(hkv), int(d), float(base), _p(k_raw, _u16p),
                                       _p(pos, _i32p), _p(out, _u16p))
    if rc != 0:
        raise RuntimeError(f"oracle_rope_rows_bf16 failed with status {rc}")
    return out
