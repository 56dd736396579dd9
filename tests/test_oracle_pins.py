"""Pins for the fp64 oracle, independent of its own code.

Each check ties the oracle to something the pages or mathematics fix, not to
a re-typed copy of its formulas:
  * scores against a brute-force loop over the RELATIVE-angle closed form of
    RoPE attention (gist.science, "LazyAttention: Efficient Retrieval-
    Augmented Generation with Deferred Positional Encoding", Technical
    Summary: Mathematical Equivalence -- scores depend only on n - m);
  * invariance of outputs under a common shift of every position (same
    passage);
  * equality with ordinary causal attention when documents sit contiguously
    (prefix reuse is the special case of contiguous placement; abstract and
    Problem Statement), computed with torch's float64 SDPA and complex-number
    RoPE;
  * softmax invariants (constant values reproduce themselves, a single
    visible key returns its value exactly, no visible key gives zeros);
  * bf16 rounding against torch's float32 -> bf16 conversion and hand ties;
  * the table-word codec against hand-computed words;
  * ALiBi (Key Contributions: the method extends to other relative
    encodings): the default head slopes against values derived by hand from
    the ALiBi paper's rule; with identical keys every score is the same up to
    the bias, so each head's output is a geometric-weight average with a
    closed form; equality with torch's float64 SDPA given the bias as an
    additive mask on contiguous placements; shift invariance.
"""
import numpy as np
import pytest
import torch

import oracle
from tests._cases import bits_to_f64, make_case

D = 16
BASE = 500000.0


def _theta(d, base):
    return base ** (-(2.0 * np.arange(d // 2)) / d)


def _brute_scores_and_out(case):
    """Per (query, head) row: scores from the relative closed form, then softmax and PV."""
    d, G = case.d, case.hq // case.hkv
    th = _theta(d, case.base)
    h2 = d // 2
    rows_s, rows_o = [], []
    for r in range(case.cu_q.size - 1):
        keys = []
        for g in range(case.seg_indptr[r], case.seg_indptr[r + 1]):
            for j in range(case.seg_len[g]):
                keys.append((case.seg_src[g] + j, case.seg_off[g] + j))
        for q in range(case.cu_q[r], case.cu_q[r + 1]):
            p = int(case.q_pos[q])
            for h in range(case.hq):
                kvh = h // G
                qv = bits_to_f64(case.q_raw[q, h])
                s = np.full(len(keys), -np.inf)
                for u, (row, pos) in enumerate(keys):
                    if pos > p:
                        continue
                    kv = bits_to_f64(case.k_tok[row, kvh])
                    qa, qb, ka, kb = qv[:h2], qv[h2:], kv[:h2], kv[h2:]
                    ang = (p - pos) * th
                    s[u] = np.sum((qa * ka + qb * kb) * np.cos(ang) - (qb * ka - qa * kb) * np.sin(ang)) / np.sqrt(d)
                o = np.zeros(d)
                if np.isfinite(s).any():
                    w = np.exp(s - s[np.isfinite(s)].max())
                    w[~np.isfinite(s)] = 0
                    vals = np.stack([bits_to_f64(case.v_tok[row, kvh]) for row, _ in keys])
                    o = (w[:, None] * vals).sum(0) / w.sum()
                rows_s.append(s)
                rows_o.append(o)
    return rows_s, np.array(rows_o)


def _adversarial_case(seed=7, hq=4, hkv=2):
    # request 0: two documents with a gap, the SAME document (store rows 0..9)
    # placed twice at different offsets, a partial question; request 1: a
    # single short document, queries before, inside and after it.
    reqs = [
        ([(0, 0, 10), (10, 25, 7), (0, 40, 10), (17, 50, 5)], [50, 52, 54, 60]),
        ([(22, 3, 6)], [0, 3, 5, 8, 100]),
    ]
    return make_case(seed, hq=hq, hkv=hkv, d=D, requests=reqs)


@pytest.mark.parametrize("hq,hkv", [(4, 2), (4, 1), (2, 2), (8, 2)])
def test_scores_match_relative_closed_form(hq, hkv):
    case = _adversarial_case(hq=hq, hkv=hkv)
    out, scores = oracle.attend(**case.oracle_kwargs(), want_scores=True)
    bs, bo = _brute_scores_and_out(case)
    for i, s in enumerate(bs):
        o_s = scores[i, :s.size]
        assert np.array_equal(np.isinf(o_s), np.isinf(s)), f"mask differs on row {i}"
        fin = np.isfinite(s)
        np.testing.assert_allclose(o_s[fin], s[fin], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out, bo, rtol=1e-12, atol=1e-13)


def test_shift_invariance():
    case = _adversarial_case()
    out0 = oracle.attend(**case.oracle_kwargs())
    for c in (1, 977, 12345):
        kw = case.oracle_kwargs()
        kw["seg_off"] = case.seg_off + c
        kw["q_pos"] = case.q_pos + c
        out = oracle.attend(**kw)
        np.testing.assert_allclose(out, out0, rtol=1e-10, atol=1e-11)


def _rope_complex(x, pos, base):
    """RoPE via complex multiplication of the rotate-half pairs (x_i + i x_{i+d/2})."""
    d = x.shape[-1]
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    z = z * np.exp(1j * np.multiply.outer(pos, _theta(d, base)))[..., None, :] if np.ndim(pos) else z * np.exp(1j * pos * _theta(d, base))
    return np.concatenate([z.real, z.imag], axis=-1)


@pytest.mark.parametrize("hq,hkv", [(4, 2), (6, 3), (4, 4)])
def test_contiguous_placement_equals_prefix_attention(hq, hkv):
    lens = [9, 13, 6]
    offs = np.cumsum([0] + lens[:-1])
    segs = []
    row = 0
    for o, L in zip(offs, lens):
        segs.append((row, int(o), L))
        row += L
    total = sum(lens)
    qp = list(range(total - 6, total))  # the last segment plays the question
    case = make_case(11, hq=hq, hkv=hkv, d=D, requests=[(segs, qp)])
    out = oracle.attend(**case.oracle_kwargs())
    # ordinary causal attention over one concatenated sequence, absolute RoPE
    pos = np.arange(total)
    k = _rope_complex(bits_to_f64(case.k_tok[:total]), pos, BASE)   # [T, Hkv, d]
    v = bits_to_f64(case.v_tok[:total])
    q = _rope_complex(bits_to_f64(case.q_raw), np.array(qp), BASE)   # [Tq, Hq, d]
    G = hq // hkv
    K = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(G, 0)
    V = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(G, 0)
    Q = torch.from_numpy(q).permute(1, 0, 2)
    mask = torch.from_numpy(pos[None, :] <= np.array(qp)[:, None])
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask)
    ref = ref.permute(1, 0, 2).reshape(-1, D).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_constant_values_reproduce_and_rows_sum_to_one():
    case = _adversarial_case()
    c = 0x3FC0  # bf16 1.5
    case.v_tok[:] = c
    out = oracle.attend(**case.oracle_kwargs())
    G = case.hq // case.hkv
    for i in range(out.shape[0]):
        q = i // case.hq
        r = int(np.searchsorted(case.cu_q, q, side="right") - 1)
        has_key = any(case.seg_off[g] <= case.q_pos[q]
                      for g in range(case.seg_indptr[r], case.seg_indptr[r + 1]))
        expect = 1.5 if has_key else 0.0
        np.testing.assert_allclose(out[i], expect, rtol=1e-14, atol=0)
    assert G >= 1


def test_single_visible_key_returns_its_value_and_none_gives_zero():
    # one segment at offset 5; a query at 5 sees only key j=0, one at 4 sees none
    case = make_case(3, hq=2, hkv=1, d=D, requests=[([(0, 5, 4)], [5, 4])])
    out = oracle.attend(**case.oracle_kwargs())
    v0 = bits_to_f64(case.v_tok[0, 0])
    assert np.array_equal(out[0], v0) and np.array_equal(out[1], v0)
    assert np.array_equal(out[2], np.zeros(D)) and np.array_equal(out[3], np.zeros(D))


def test_decode_row_equals_last_prefill_row():
    segs = [(0, 0, 20), (20, 20, 12)]
    case = make_case(5, hq=4, hkv=2, d=D, requests=[(segs, list(range(20, 32)))])
    full = oracle.attend(**case.oracle_kwargs())
    kw = case.oracle_kwargs()
    kw.update(q_raw=case.q_raw[-1:], cu_q=np.array([0, 1], np.int32), q_pos=case.q_pos[-1:])
    last = oracle.attend(**kw)
    np.testing.assert_array_equal(full[-4:], last)


def test_selected_rows_equal_full_rows():
    case = _adversarial_case()
    full = oracle.attend(**case.oracle_kwargs())
    sel = np.array([0, 5, 17, 30, 35])
    out = oracle.attend(**case.oracle_kwargs(), sel_q=sel // case.hq, sel_h=sel % case.hq)
    np.testing.assert_array_equal(out, full[sel])


# --------------------------------------------------------------------------- rope
def test_rope_matches_complex_rotation_and_composes():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(128)
    for pos in (0, 1, 17, 4160, 32767):
        y = oracle.rope(x, pos, BASE)
        np.testing.assert_allclose(y, _rope_complex(x, pos, BASE), rtol=0, atol=1e-12)
        np.testing.assert_allclose(np.linalg.norm(y), np.linalg.norm(x), rtol=1e-14)
    assert np.array_equal(oracle.rope(x, 0, BASE), x)
    np.testing.assert_allclose(oracle.rope(oracle.rope(x, 300, BASE), 4000, BASE),
                               oracle.rope(x, 4300, BASE), atol=1e-11)


# --------------------------------------------------------------------------- bf16
def test_bf16_rounding_matches_torch_on_float32_values():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(4000), rng.standard_normal(1000) * 1e-3,
                        rng.standard_normal(1000) * 1e4]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.f64_to_bf16(x.astype(np.float64)), ref)


def test_bf16_rounding_ties_and_single_rounding():
    one = 0x3F80
    assert oracle.f64_to_bf16(np.array([1.0 + 2.0 ** -8]))[0] == one          # tie -> even (1.0)
    assert oracle.f64_to_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == one + 2  # tie -> even (1+2^-6)
    # just above a tie by less than a float32 ulp: a double->float->bf16 path
    # would see an exact tie and round down; one rounding step rounds up.
    assert oracle.f64_to_bf16(np.array([1.0 + 2.0 ** -8 + 2.0 ** -30]))[0] == one + 1
    assert oracle.f64_to_bf16(np.array([-2.0]))[0] == 0xC000
    assert np.array_equal(oracle.bf16_to_f64(np.array([0x3F80, 0xC000, 0x0000], np.uint16)), [1.0, -2.0, 0.0])


# --------------------------------------------------------------------------- codec
def test_word_codec_hand_values_and_limits():
    assert oracle.pack_word(0, 0) == 0
    assert oracle.pack_word(1, 0) == 1
    assert oracle.pack_word(0, 1) == 131072
    assert oracle.pack_word(131071, 32767) == 0xFFFFFFFF
    assert oracle.pack_word(5, 100) == 100 * 131072 + 5
    for b, o in [(0, 0), (131071, 0), (0, 32767), (131071, 32767), (12345, 4160)]:
        assert oracle.unpack_word(oracle.pack_word(b, o)) == (b, o)
    for b, o in [(131072, 0), (0, 32768), (-1, 0), (0, -1)]:
        with pytest.raises(ValueError):
            oracle.pack_word(b, o)


def test_expand_table_hand_example():
    meta = np.zeros(8, np.uint32)
    meta[5] = oracle.pack_meta(2, 10)   # third block of its segment, 10 slots written
    meta[1] = oracle.pack_meta(0, 16)
    words = np.array([oracle.pack_word(5, 100), oracle.pack_word(1, 7)], np.uint32)
    blk, slot, pos, rc = oracle.expand_table(words, meta, 8)
    assert rc == 0
    assert (blk[0] == 5).all() and (blk[1] == 1).all()
    assert list(slot[0]) == list(range(80, 96)) and list(slot[1]) == list(range(16, 32))
    assert list(pos[0]) == [100 + 32 + s for s in range(10)] + [-1] * 6
    assert list(pos[1]) == list(range(7, 23))
    _, _, _, rc = oracle.expand_table(np.array([oracle.pack_word(9, 0)], np.uint32), meta, 8)
    assert rc == -2


# --------------------------------------------------------------------------- pool writes
def test_kv_write_expected_pool():
    rng = np.random.default_rng(2)
    hkv, d, nb = 2, 128, 6
    from position_agnostic_paged_b200.workloads import randn_bf16
    n = 40
    k = randn_bf16(rng, (n, hkv, d))
    v = randn_bf16(rng, (n, hkv, d))
    # a 40-token segment placed in blocks 3,4,5 (local j = 0..39 -> blocks 3 + j//16)
    j = np.arange(n, dtype=np.int32)
    slot = (3 * 16 + j).astype(np.int32)
    kp = np.full((nb, hkv, 16, d), 0xFFFF, np.uint16)
    vp = np.full((nb, hkv, 16, d), 0xFFFF, np.uint16)
    meta = np.zeros(nb, np.uint32)
    assert oracle.kv_write(k, v, slot, j, kp, vp, meta, BASE) == 0
    # untouched blocks keep the sentinel
    assert (kp[:3] == 0xFFFF).all() and (vp[:3] == 0xFFFF).all()
    # values copied verbatim, j = 0 is the identity rotation
    assert np.array_equal(vp[3:].reshape(-1, hkv, 16, d).transpose(0, 2, 1, 3).reshape(-1, hkv, d)[:n], v)
    assert np.array_equal(kp[3, :, 0], k[0])
    # rotated keys are the correctly rounded complex rotation (half a bf16 ulp)
    got = bits_to_f64(kp[3:].transpose(0, 2, 1, 3).reshape(-1, hkv, d)[:n])
    exact = _rope_complex(bits_to_f64(k), j.astype(np.float64), BASE)
    err = np.abs(got - exact)
    assert (err <= np.abs(exact) * 2.0 ** -8 + 1e-30).all()
    assert list(meta[3:]) == [oracle.pack_meta(0, 16), oracle.pack_meta(1, 16), oracle.pack_meta(2, 8)]
    # a token whose local index is not congruent to its slot is rejected
    assert oracle.kv_write(k[:1], v[:1], np.array([3 * 16 + 1], np.int32), np.array([0], np.int32),
                           kp, vp, meta, BASE) == -2


def test_rope_rows_bf16_matches_rotation():
    rng = np.random.default_rng(4)
    from position_agnostic_paged_b200.workloads import randn_bf16
    k = randn_bf16(rng, (5, 2, 128))
    pos = np.array([0, 1, 513, 4160, 20000], np.int32)
    out = oracle.rope_rows_bf16(k, pos, BASE)
    assert np.array_equal(out[0], k[0])
    exact = _rope_complex(bits_to_f64(k), pos.astype(np.float64), BASE)
    assert (np.abs(bits_to_f64(out) - exact) <= np.abs(exact) * 2.0 ** -8 + 1e-30).all()


# ----------------------------------------------------------------------------- RoPE frequency tables
def test_llama31_table_regions_by_hand():
    """base 5e5, d 128, factor 8, low/high factors 1/4, original context 8192.  A component keeps its
    frequency when its wavelength 2*pi*5e5^(i/64) is below 8192/4 = 2048, i.e. 5e5^(i/64) < 325.95,
    i < 64*ln(325.95)/ln(5e5) = 28.22 -> i = 0..28; it is divided by 8 when the wavelength exceeds
    8192, i.e. i > 64*ln(1303.8)/ln(5e5) = 34.99 -> i = 35..63; i = 29..34 are interpolated."""
    th = oracle.llama31_theta(500000.0, 128, 8.0, 1.0, 4.0, 8192.0)
    plain = np.array([500000.0 ** (-i / 64.0) for i in range(64)])
    assert np.array_equal(th[:29], plain[:29])
    np.testing.assert_allclose(th[35:], plain[35:] / 8.0, rtol=0, atol=0)
    mid = th[29:35] / plain[29:35]
    assert np.all(mid < 1.0) and np.all(mid > 1.0 / 8.0)
    assert np.all(np.diff(th) < 0)                      # frequencies still decrease with i


def test_llama31_table_factor_one_and_continuity():
    plain = oracle.llama31_theta(10000.0, 64, 1.0, 1.0, 4.0, 2048.0)
    np.testing.assert_allclose(plain, [10000.0 ** (-2.0 * i / 64) for i in range(32)], rtol=1e-15)
    # a frequency sitting exactly on either boundary gets the same value from both sides
    import math
    base, d, orig = 500000.0, 128, 8192.0
    for wl_edge, expect_ratio in ((orig / 4.0, 1.0), (orig / 1.0, 1.0 / 8.0)):
        # choose base so that component 1 has exactly that wavelength
        f = 2 * math.pi / wl_edge
        b = f ** (-d / 2.0)
        th = oracle.llama31_theta(b, d, 8.0, 1.0, 4.0, orig)
        assert abs(th[1] / f - expect_ratio) < 1e-12


def test_rope_with_a_table_is_relative_and_default_table_matches():
    rng = np.random.default_rng(5)
    q = rng.standard_normal(128)
    k = rng.standard_normal(128)
    th = oracle.llama31_theta()
    s1 = oracle.rope(q, 9000, 500000.0, theta=th) @ oracle.rope(k, 1234, 500000.0, theta=th)
    s2 = oracle.rope(q, 9000 + 77777, 500000.0, theta=th) @ oracle.rope(k, 1234 + 77777, 500000.0, theta=th)
    assert abs(s1 - s2) < 1e-9 * max(1.0, abs(s1))
    dflt = np.array([500000.0 ** (-2.0 * i / 128) for i in range(64)])
    np.testing.assert_array_equal(oracle.rope(q, 4321, 500000.0, theta=dflt), oracle.rope(q, 4321, 500000.0))
    # and the scaled table really changes long-wavelength components
    assert not np.allclose(oracle.rope(q, 4321, 500000.0, theta=th), oracle.rope(q, 4321, 500000.0))


# --------------------------------------------------------------------------- ALiBi
def alibi_pin_slopes_by_hand(lib=None):
    # the rule: n a power of two -> 2^(-8k/n), k = 1..n; otherwise the 2^m < n slopes, then the
    # even-position terms of the 2^(m+1) sequence
    want = {1: [-8.0], 2: [-4.0, -8.0], 8: list(-np.arange(1.0, 9.0)), 6: [-2.0, -4.0, -6.0, -8.0, -1.0, -3.0],
            12: [-1.0, -2.0, -3.0, -4.0, -5.0, -6.0, -7.0, -8.0, -0.5, -1.5, -2.5, -3.5]}
    for n, e in want.items():
        np.testing.assert_allclose(oracle.alibi_slopes(n, lib=lib), 2.0 ** np.array(e), rtol=1e-15, atol=0)


def alibi_pin_geometric_weights(lib=None):
    # every key the same vector: q.k is one constant per (query, head), so the weights are
    # exp(-m_h (p - t)) / sum, a geometric sequence in the distance; component 0 of the output is
    # then the weighted mean of the values' component 0 over the visible keys
    case = _adversarial_case(hq=4, hkv=2)
    case.k_tok[:] = case.k_tok[0:1]
    slopes = np.array([0.5, 0.125, 0.03, 0.9])
    out = oracle.attend(**case.oracle_kwargs(), alibi_slopes=slopes, lib=lib)
    G = case.hq // case.hkv
    i = 0
    for r in range(case.cu_q.size - 1):
        keys = [(case.seg_src[g] + j, case.seg_off[g] + j)
                for g in range(case.seg_indptr[r], case.seg_indptr[r + 1]) for j in range(case.seg_len[g])]
        for q in range(case.cu_q[r], case.cu_q[r + 1]):
            p = int(case.q_pos[q])
            for h in range(case.hq):
                vis = [(row, pos) for row, pos in keys if pos <= p]
                if not vis:
                    assert np.all(out[i] == 0)
                else:
                    w = np.array([np.exp(-slopes[h] * (p - pos)) for _, pos in vis])
                    v0 = np.array([bits_to_f64(case.v_tok[row, h // G])[0] for row, _ in vis])
                    np.testing.assert_allclose(out[i, 0], (w * v0).sum() / w.sum(), rtol=1e-12, atol=1e-13)
                i += 1


def alibi_pin_contiguous_equals_sdpa(lib=None):
    lens = [9, 13, 6]
    segs, row = [], 0
    for o, L in zip(np.cumsum([0] + lens[:-1]), lens):
        segs.append((row, int(o), L))
        row += L
    total = sum(lens)
    qp = np.arange(total - 6, total)
    hq, hkv = 6, 3
    case = make_case(12, hq=hq, hkv=hkv, d=D, requests=[(segs, list(qp))])
    slopes = oracle.alibi_slopes(hq, lib=lib)
    out = oracle.attend(**case.oracle_kwargs(), alibi_slopes=slopes, lib=lib)
    # no rotation; the bias as an additive float mask, -inf where the key is in the future
    G = hq // hkv
    K = torch.from_numpy(bits_to_f64(case.k_tok[:total])).permute(1, 0, 2).repeat_interleave(G, 0)
    V = torch.from_numpy(bits_to_f64(case.v_tok[:total])).permute(1, 0, 2).repeat_interleave(G, 0)
    Q = torch.from_numpy(bits_to_f64(case.q_raw)).permute(1, 0, 2)
    dist = qp[:, None] - np.arange(total)[None, :]
    bias = -slopes[:, None, None] * dist[None]
    bias = np.where(dist[None] >= 0, bias, -np.inf)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=torch.from_numpy(bias))
    np.testing.assert_allclose(out, ref.permute(1, 0, 2).reshape(-1, D).numpy(), rtol=1e-12, atol=1e-13)
    # slopes of zero: plain causal attention without any positional encoding
    out0 = oracle.attend(**case.oracle_kwargs(), alibi_slopes=np.zeros(hq), lib=lib)
    ref0 = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=torch.from_numpy(dist >= 0))
    np.testing.assert_allclose(out0, ref0.permute(1, 0, 2).reshape(-1, D).numpy(), rtol=1e-12, atol=1e-13)


def alibi_pin_shift_invariance(lib=None):
    case = _adversarial_case()
    slopes = oracle.alibi_slopes(case.hq, lib=lib)
    out0 = oracle.attend(**case.oracle_kwargs(), alibi_slopes=slopes, lib=lib)
    for c in (1, 977, 12345):
        kw = case.oracle_kwargs()
        kw["seg_off"] = case.seg_off + c
        kw["q_pos"] = case.q_pos + c
        np.testing.assert_allclose(oracle.attend(**kw, alibi_slopes=slopes, lib=lib), out0, rtol=1e-10, atol=1e-11)


ALIBI_PINS = [alibi_pin_slopes_by_hand, alibi_pin_geometric_weights, alibi_pin_contiguous_equals_sdpa,
              alibi_pin_shift_invariance]


@pytest.mark.parametrize("pin", ALIBI_PINS, ids=lambda f: f.__name__)
def test_alibi(pin):
    pin()


def test_alibi_needs_one_slope_per_query_head_and_leaves_rope_calls_alone():
    case = _adversarial_case()
    with pytest.raises(ValueError):
        oracle.attend(**case.oracle_kwargs(), alibi_slopes=np.ones(case.hq + 1))
    a = oracle.attend(**case.oracle_kwargs())
    oracle.attend(**case.oracle_kwargs(), alibi_slopes=np.ones(case.hq))
    assert np.array_equal(oracle.attend(**case.oracle_kwargs()), a)
