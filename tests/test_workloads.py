"""The synthetic input recipe: the configurations' shapes, placements and skew, seeded and
deterministic.  Both the oracle and the CUDA path read these inputs, so the recipe is pinned here
against the stated configurations (documents placed contiguously in random order, the question
after them, Zipf draws without replacement within a request)."""
import numpy as np

from position_agnostic_paged_b200 import accounting
from position_agnostic_paged_b200 import workloads as W


def _segments(step, r):
    g0, g1 = step.seg_indptr[r], step.seg_indptr[r + 1]
    return step.seg_src[g0:g1], step.seg_off[g0:g1], step.seg_len[g0:g1]


def _check_contiguous(off, ln):
    assert off[0] == 0 and np.array_equal(off[1:], np.cumsum(ln)[:-1])


def test_decode_8b_recipe():
    wl = W.make("decode_8b")
    assert (wl.hq, wl.hkv, wl.d) == (32, 8, 128)
    (step,) = wl.steps
    assert step.kind == "decode" and step.num_req == 64
    assert np.all(step.kv_len == 4161) and np.all(step.q_pos == 4160)
    tops = []
    for r in range(step.num_req):
        src, off, ln = _segments(step, r)
        assert list(ln) == [512] * 8 + [65]            # 8 documents, 64-token question + the new token
        _check_contiguous(off, ln)
        assert len(set(src[:8].tolist())) == 8            # distinct documents within a request
        tops.extend(src[:8].tolist())
    # Zipf(1.0) over 1000 documents: the most popular document is in most requests
    counts = np.unique(tops, return_counts=True)[1]
    assert counts.max() >= 32
    assert accounting.decode_kv_bytes(step.kv_len, wl.hkv, wl.d) == 64 * 4161 * 4096


def test_prefill_8b_recipe():
    wl = W.make("prefill_8b")
    (step,) = wl.steps
    assert step.kind == "prefill" and step.num_req == 16 and step.total_q == 16 * 256
    for r in range(step.num_req):
        src, off, ln = _segments(step, r)
        assert list(ln) == [512] * 10 + [256]
        _check_contiguous(off, ln)
        assert len(set(src[:10].tolist())) == 10
        assert np.array_equal(step.q_pos[step.cu_q[r]:step.cu_q[r + 1]], 5120 + np.arange(256))
    # visible (query, key) pairs per head: 256 x 5120 document keys plus the causal chunk
    assert step.visible_pairs == 16 * (256 * 5120 + 256 * 257 // 2) == 16 * 1343616


def test_tiny_recipe():
    wl = W.make("tiny")
    assert (wl.hq, wl.hkv) == (8, 2)
    kinds = [st.kind for st in wl.steps]
    assert kinds == ["prefill"] + ["decode"] * 4
    pf = wl.steps[0]
    src, off, ln = _segments(pf, 0)
    assert list(off) == [0, 256, 512, 768] and list(ln) == [256, 256, 256, 64]
    assert len(set(src[:3].tolist())) == 3
    assert np.array_equal(pf.q_pos, 768 + np.arange(64))
    for i, st in enumerate(wl.steps[1:]):
        assert st.q_pos.tolist() == [832 + i]
        assert int(st.kv_len[0]) == 833 + i            # each decode writes its token first


def test_mixed_8b_recipe():
    wl = W.make("mixed_8b")
    # the pool is capped at 1 GiB: blocks x Hkv x 16 tokens x 128 x 2 bytes x (K, V)
    assert wl.num_blocks * wl.hkv * 16 * 128 * 2 * 2 == 1 << 30
    by = {st.kind: st for st in wl.steps}
    pf, dc = by["prefill"], by["decode"]
    assert pf.num_req == 32 and pf.total_q == 32 * 256 and dc.num_req == 192
    for st, n_docs, tail in ((pf, 10, 256), (dc, 8, 65)):
        for r in range(0, st.num_req, 7):
            src, off, ln = _segments(st, r)
            assert len(ln) == n_docs + 1 and ln[-1] == tail
            assert np.all((ln[:-1] >= 128) & (ln[:-1] <= 2048))
            _check_contiguous(off, ln)


def test_inputs_are_seeded_and_deterministic():
    a, b = W.make("decode_8b"), W.make("decode_8b")
    sa, sb = a.steps[0], b.steps[0]
    assert np.array_equal(sa.q_raw, sb.q_raw) and np.array_equal(sa.table_block, sb.table_block)
    assert np.array_equal(sa.seg_src, sb.seg_src) and np.array_equal(a.k_store[:4096], b.k_store[:4096])
    c = W.make("decode_8b", seed=7)
    assert not np.array_equal(c.steps[0].seg_src, sa.seg_src)


def test_distinct_decode_workload_shares_no_document():
    """decode_8b_distinct: the decode 8B shapes with every document in exactly one request, so the
    step's logical K/V bytes are all distinct physical bytes."""
    wl = W.make("decode_8b_distinct", n_decode=8)
    st = wl.steps[0]
    seen = set()
    for r in range(st.num_req):
        blocks = set(st.table_block[st.table_indptr[r]:st.table_indptr[r + 1]].tolist())
        assert not (blocks & seen)
        seen |= blocks
    assert wl.info["unique_docs_used"] == 8 * 8
    assert (st.kv_len == 8 * 512 + 65).all()
