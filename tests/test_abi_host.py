"""The C-ABI library loads, exports every symbol its header declares, and its
host-side logic (word codec, argument validation, workspace sizing) behaves as
documented.  Nothing here launches a kernel, so it runs without a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from position_agnostic_paged_b200 import lazy_attn as la

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "lazy_attn.h")


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?(?:int|size_t|char\s*\*|void|lazy_block_cache)\s*\*?\s*(lazy_\w+)\s*\(",
                       txt, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 12
    lib = ctypes.CDLL(la.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in lazy_attn.h but not exported"
    assert sorted(la.EXPORTED) == names


def test_version_and_strerror():
    assert la.version() == 102
    for code in (0, -1, -2, -3, -4, -5):
        assert la.strerror(code) and la.strerror(code) != "unknown error"


def test_pack_words_bit_exact_against_oracle():
    rng = np.random.default_rng(0)
    b = np.concatenate([[0, 131071, 0, 131071], rng.integers(0, 131072, 1000)]).astype(np.int32)
    o = np.concatenate([[0, 0, 32767, 32767], rng.integers(0, 32768, 1000)]).astype(np.int32)
    got = la.pack_words(b, o)
    ref = np.array([oracle.pack_word(int(x), int(y)) for x, y in zip(b, o)], np.uint32)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("b,o", [(131072, 0), (0, 32768), (-1, 0), (0, -5)])
def test_pack_words_rejects_overflow(b, o):
    with pytest.raises(la.LazyAttnError) as e:
        la.pack_words(np.array([1, b], np.int32), np.array([1, o], np.int32))
    assert e.value.code == la.LAZY_ERANGE


def _call_decode(cfg, **kw):
    c = cfg.c()
    args = dict(q=1, qp=1, n=2, table=1, indptr=1, maxw=4, meta=1, k=1, v=1, nb=8, out=1, ws=1, wsb=1 << 20)
    args.update(kw)
    return la._lib.lazy_decode_attn(ctypes.byref(c), args["q"], args["qp"], args["n"], args["table"],
                                    args["indptr"], args["maxw"], args["meta"], args["k"], args["v"], args["nb"],
                                    args["out"], args["ws"], args["wsb"], None, None)


def test_host_validation_returns_before_launch():
    ok = la.Cfg(8, 2)
    assert _call_decode(la.Cfg(8, 2, head_dim=64)) == la.LAZY_ESHAPE
    assert _call_decode(la.Cfg(8, 3)) == la.LAZY_ESHAPE
    assert _call_decode(la.Cfg(64, 1)) == la.LAZY_ESHAPE          # G = 64 > 32
    assert _call_decode(la.Cfg(8, 2, block_size=32)) == la.LAZY_ESHAPE
    assert _call_decode(ok, q=None) == la.LAZY_EINVAL
    assert _call_decode(ok, n=-1) == la.LAZY_EINVAL
    assert _call_decode(ok, nb=(1 << 17) + 1) == la.LAZY_ERANGE
    assert _call_decode(ok, wsb=16) == la.LAZY_EWORKSPACE
    assert _call_decode(ok, ws=None) == la.LAZY_EWORKSPACE
    c = ok.c()
    assert la._lib.lazy_kv_write(None, 1, 1, 1, 1, 1, 1, 1, 1, 8, None, None) == la.LAZY_EINVAL
    assert la._lib.lazy_kv_write(ctypes.byref(c), None, 1, 1, 1, 1, 1, 1, 1, 8, None, None) == la.LAZY_EINVAL
    assert la._lib.lazy_materialize_k(ctypes.byref(c), None, 4, 1, 1, 8, 1, None, None) == la.LAZY_EINVAL
    assert la._lib.lazy_debug_decode_table(None, 4, 1, 8, 1, 1, 1, None, None) == la.LAZY_EINVAL


def test_decode_workspace_sizes():
    cfg = la.Cfg(32, 8)
    a = la.decode_workspace_bytes(cfg, 64, 261)
    b = la.decode_workspace_bytes(cfg, 1, 261)
    assert 0 < b < a
    # one (m, l, acc[128]) record of fp32 per (request, kv head, split, head in group)
    assert a % ((128 + 2) * 4 * 4) == 0
    assert la.decode_workspace_bytes(la.Cfg(32, 8, head_dim=64), 64, 261) == 0


def test_alibi_validation_returns_before_launch():
    sl = tuple([0.25] * 8)
    assert _call_decode(la.Cfg(256, 8, alibi_slopes=tuple([0.1] * 256))) == la.LAZY_ESHAPE   # Hq > 128
    assert _call_decode(la.Cfg(8, 2, alibi_slopes=(float("nan"),) + sl[1:])) == la.LAZY_EINVAL
    assert _call_decode(la.Cfg(8, 2, alibi_slopes=(float("inf"),) + sl[1:])) == la.LAZY_EINVAL
    c = la.Cfg(8, 2, alibi_slopes=sl).c()
    # the stored keys carry no position: materialisation and the plain paths refuse ALiBi
    assert la._lib.lazy_materialize_k(ctypes.byref(c), 1, 4, 1, 1, 8, 1, None, None) == la.LAZY_EINVAL
    assert la._lib.lazy_plain_decode_attn(ctypes.byref(c), 1, 1, 2, 1, 1, 4, 1, 1, 8, 1, 8, 1, 1, 1 << 20,
                                          None, None) == la.LAZY_EINVAL
    assert la._lib.lazy_plain_prefill_attn(ctypes.byref(c), 1, 1, 1, 1, 4, 4, 1, 1, 4, 1, 1, 8, 1, 8, 1, 1,
                                           1 << 20, None, None) == la.LAZY_EINVAL
    with pytest.raises(ValueError):
        la.Cfg(8, 2, alibi_slopes=sl[:4]).c()


def test_alibi_slopes_helper_by_hand():
    from position_agnostic_paged_b200.rope import alibi_slopes
    np.testing.assert_allclose(alibi_slopes(8), 2.0 ** -np.arange(1.0, 9.0), rtol=1e-15, atol=0)
    np.testing.assert_allclose(np.log2(alibi_slopes(12)), [-1, -2, -3, -4, -5, -6, -7, -8, -0.5, -1.5, -2.5, -3.5],
                               rtol=0, atol=1e-13)
    with pytest.raises(ValueError):
        alibi_slopes(0)


def test_mixed_step_validates_both_batches_before_launching():
    c = la.Cfg(8, 2).c()
    pf = la.PrefillBatch(1, 1, 1, 2, 8, 4, 1, 1, 4, 1, 1, 1 << 20)
    same_ws = la.DecodeBatch(1, 1, 2, 1, 1, 4, 1, 1, 1 << 20)
    small_ws = la.DecodeBatch(1, 1, 2, 1, 1, 4, 1, 2, 16)
    call = lambda cfg, p, d: la._lib.lazy_mixed_attn(ctypes.byref(cfg), ctypes.byref(p) if p else None,
                                                    ctypes.byref(d) if d else None, 1, 1, 1, 8, None, None)
    assert call(c, pf, same_ws) == la.LAZY_EINVAL          # one workspace for both batches
    assert call(c, pf, small_ws) == la.LAZY_EWORKSPACE     # the decode batch fails: nothing launched
    assert call(la.Cfg(8, 3).c(), pf, small_ws) == la.LAZY_ESHAPE
    assert call(c, None, None) == la.LAZY_OK              # nothing to do
    bad_pf = la.PrefillBatch(1, 1, 1, 2, -1, 4, 1, 1, 4, 1, 1, 1 << 20)
    assert call(c, bad_pf, la.DecodeBatch(1, 1, 2, 1, 1, 4, 1, 3, 1 << 20)) == la.LAZY_EINVAL


def test_position_tables_agree_with_the_oracle_s_own():
    """The library's RoPE-variant and ALiBi tables and the oracle's are two independent
    computations of the published rules; they must agree."""
    from position_agnostic_paged_b200 import rope
    np.testing.assert_allclose(rope.llama31_theta(), oracle.llama31_theta(), rtol=1e-14, atol=0)
    np.testing.assert_allclose(rope.default_theta(), 500000.0 ** (-(2.0 * np.arange(64)) / 128), rtol=1e-15)
    for n in (1, 2, 3, 5, 6, 8, 12, 16, 24, 32, 40, 64, 96, 128):
        np.testing.assert_allclose(rope.alibi_slopes(n), oracle.alibi_slopes(n), rtol=1e-14, atol=0)


def test_table_exports_against_the_oracle_over_parameters():
    """lazy_rope_theta, lazy_rope_theta_llama31 and lazy_alibi_slopes called through the C ABI
    against the oracle's own computations, over bases, head sizes and scaling parameters."""
    for base, d in ((500000.0, 128), (10000.0, 64), (1.0e6, 256), (2.5, 8)):
        np.testing.assert_allclose(la.rope_theta(base, d), base ** (-(2.0 * np.arange(d // 2)) / d),
                                   rtol=1e-15, atol=0)
    for args in ((500000.0, 128, 8.0, 1.0, 4.0, 8192.0), (10000.0, 64, 4.0, 1.0, 4.0, 2048.0),
                 (500000.0, 128, 1.0, 1.0, 4.0, 8192.0), (1.0e6, 128, 32.0, 2.0, 8.0, 65536.0)):
        np.testing.assert_allclose(la.rope_theta_llama31(*args), oracle.llama31_theta(*args), rtol=1e-14, atol=0)
    for n in range(1, 129):
        np.testing.assert_allclose(la.alibi_slopes(n), oracle.alibi_slopes(n), rtol=1e-14, atol=0)
    # arguments outside each rule's domain are refused before anything is written
    buf = np.full(64, 7.0)
    for bad in ((1.0, 128), (500000.0, 127), (500000.0, 0), (float("nan"), 128)):
        assert la._lib.lazy_rope_theta(bad[0], bad[1], buf.ctypes.data) == la.LAZY_EINVAL
    for bad in ((500000.0, 128, 0.0, 1.0, 4.0, 8192.0), (500000.0, 128, 8.0, 4.0, 4.0, 8192.0),
                (500000.0, 128, 8.0, 1.0, 4.0, 0.0)):
        assert la._lib.lazy_rope_theta_llama31(*bad, buf.ctypes.data) == la.LAZY_EINVAL
    assert la._lib.lazy_alibi_slopes(0, buf.ctypes.data) == la.LAZY_EINVAL
    assert la._lib.lazy_alibi_slopes(4, None) == la.LAZY_EINVAL
    assert (buf == 7.0).all()


def test_header_is_plain_c_and_cxx(tmp_path):
    """The public header compiles as C99 and C++11 on its own, and its inline codec packs words as
    documented (a C program built against the header alone, no CUDA)."""
    import shutil
    import subprocess
    inc = os.path.dirname(HEADER)
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    for lang, std in (("c", "-std=c99"), ("c++", "-std=c++11")):
        cc = "gcc" if lang == "c" else "g++"
        r = subprocess.run([cc, "-x", lang, std, "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-I", inc, HEADER],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
    src = tmp_path / "t.c"
    src.write_text('#include "lazy_attn.h"\n'
                   'int main(void) {\n'
                   '  uint32_t w = lazy_pack(131071u, 32767u);\n'
                   '  return (lazy_block(w) == 131071u && lazy_offset(w) == 32767u && lazy_pack(5u, 100u) == '
                   '((100u << 17) | 5u)) ? 0 : 1;\n}\n')
    exe = tmp_path / "t"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", inc, str(src), "-o", str(exe)], check=True)
    assert subprocess.run([str(exe)]).returncode == 0
