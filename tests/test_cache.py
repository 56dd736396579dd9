"""Block cache and cache-hit simulation (host side, no GPU).

The reference LRU and policy simulation in oracle/cache_ref.py are pinned by hand-worked sequences;
the native cache (lazy_cache_*) must then reproduce the reference's hit/miss/eviction sequence on
seeded random streams, hand out disjoint in-range blocks (consecutive from the first free extent
that holds an entry), and the library's simulator must match the reference simulation exactly."""
import numpy as np
import pytest

from oracle.cache_ref import RefLRU, ref_simulate
from position_agnostic_paged_b200 import cache_sim
from position_agnostic_paged_b200.lazy_attn import BlockCache
from position_agnostic_paged_b200.workloads import cache_stream


# ----------------------------------------------------------------------------- reference pins
def test_ref_lru_hand_worked():
    c = RefLRU(10)
    seq = [("A", 4, False), ("B", 4, False), ("A", 4, True), ("C", 4, False),   # C evicts B
           ("B", 4, False),                                                   # B evicts A
           ("C", 4, True), ("A", 4, False)]                                   # A evicts B
    for key, n, hit in seq:
        assert c.access(key, n) is hit, key
    assert list(c.entries) == ["C", "A"] and c.used == 8 and c.evictions == 3
    assert c.access("huge", 11) is False and "huge" not in c.entries and c.evictions == 3
    assert c.access("D", 2) is False and c.used == 10 and c.evictions == 3     # fits the 2 free blocks
    assert c.access("E", 3) is False and list(c.entries) == ["A", "D", "E"]    # C (4) goes, 1 free left


def _one_block_docs(k):
    return np.full(k, 16, np.int64)


POLICY_PINS = [
    # docs 0, 1 of one block each; requests [0,1], [1,0], [0,1]
    ("agnostic", 100, 4), ("aware", 100, 4), ("aware_exact", 100, 2), ("prefix", 100, 2),
    # with room for two blocks only: the re-encoded copies crowd out the originals
    ("agnostic", 2, 4), ("aware", 2, 2), ("aware_exact", 2, 0), ("prefix", 2, 0),
]


@pytest.mark.parametrize("policy,cap,want_hits", POLICY_PINS)
def test_ref_policies_hand_worked(policy, cap, want_hits):
    r = ref_simulate(policy, _one_block_docs(2), [[0, 1], [1, 0], [0, 1]], cap)
    assert r["hit_blocks"] == want_hits and r["hit_blocks"] + r["miss_blocks"] == 6


def test_ref_policies_hand_worked_trace():
    # capacity 2, policy aware: [0,1] writes 0@0, 1@16; [1,0]: 1@0 re-encodes 1@16 (hit) and evicts
    # 0@0, then 0@16 finds no copy of 0 (miss) and evicts 1@16; [0,1]: 0@0 re-encodes 0@16 (hit),
    # evicting 1@0, then 1@16 finds no copy of 1 (miss)
    r = ref_simulate("aware", _one_block_docs(2), [[0, 1], [1, 0], [0, 1]], 2)
    assert r == {"hit_blocks": 2, "miss_blocks": 4, "evictions": 4}
    # the same stream at capacity 2 under prefix: (1) and (1,0) evict (0) and (0,1), so the third
    # request misses both; under aware_exact each copy is evicted two accesses after it is written,
    # before its (document, offset) comes back
    r = ref_simulate("prefix", _one_block_docs(2), [[0, 1], [1, 0], [0, 1]], 2)
    assert r == {"hit_blocks": 0, "miss_blocks": 6, "evictions": 4}
    r = ref_simulate("aware_exact", _one_block_docs(2), [[0, 1], [1, 0], [0, 1]], 2)
    assert r == {"hit_blocks": 0, "miss_blocks": 6, "evictions": 4}


def test_ref_prefix_reuse_stops_at_the_first_miss():
    # document 0 (5 blocks) never fits a 4-block cache, so (0) always misses; the chain (0,1) is
    # resident for the second request, yet it is not reused past the miss
    lens = np.array([5 * 16, 16], np.int64)
    r = ref_simulate("prefix", lens, [[0, 1], [0, 1]], 4)
    assert r["hit_blocks"] == 0 and r["miss_blocks"] == 12
    r = ref_simulate("agnostic", lens, [[0, 1], [0, 1]], 4)
    assert r["hit_blocks"] == 1


def test_ref_unlimited_capacity_closed_forms():
    # with room for everything: agnostic hits every use but the first of each document, and the
    # re-encoding aware policy hits exactly as often; the exact-offset policy hits every use but
    # the first of each (document, offset)
    lens, reqs = cache_stream(5, n_docs=60, doc_len=(16, 200), docs_per_req=4, alpha=1.0, n_requests=300)
    nblk = -(-lens // 16)
    total = int(nblk[reqs].sum())
    first_docs = int(nblk[np.unique(reqs)].sum())
    big = int(nblk.sum()) * 50
    for pol in ("agnostic", "aware"):
        assert ref_simulate(pol, lens, reqs, big)["miss_blocks"] == first_docs
    seen, want = set(), 0
    for req in reqs:
        off = 0
        for d in req:
            if (d, off) not in seen:
                seen.add((d, off))
                want += int(nblk[d])
            off += int(lens[d])
    r = ref_simulate("aware_exact", lens, reqs, big)
    assert r["miss_blocks"] == want and r["hit_blocks"] == total - want


# ----------------------------------------------------------------------------- native cache
def _free_runs(free):
    runs, i = [], 0
    while i < len(free):
        if free[i]:
            j = i
            while j < len(free) and free[j]:
                j += 1
            runs.append((i, j - i))
            i = j
        else:
            i += 1
    return runs


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_native_cache_matches_reference_and_allocates_disjoint_blocks(seed):
    rng = np.random.default_rng(seed)
    cap = int(rng.integers(20, 60))
    nkeys = 40
    size = rng.integers(1, 12, nkeys)
    size[0] = cap + 3                                   # one key never fits
    keys = rng.zipf(1.3, 3000) % nkeys
    ref = RefLRU(cap)
    nat = BlockCache(cap)
    held = {}
    try:
        for k in keys:
            k = int(k)
            n = int(size[k])
            want = ref.access(k, n)
            got, blocks = nat.access(k, n)
            assert got is want
            if n > cap:
                assert blocks is None
                continue
            if want:
                assert np.array_equal(blocks, held[k])
                continue
            # the free space the new entry was allocated from: all but the other resident entries
            free = np.ones(cap, bool)
            for kk in ref.entries:
                if kk != k:
                    free[held[kk]] = False
            assert len(set(blocks.tolist())) == n and blocks.min() >= 0 and blocks.max() < cap
            assert free[blocks].all()
            fits = [s for s, ln in _free_runs(free) if ln >= n]
            if fits:
                assert np.array_equal(blocks, np.arange(fits[0], fits[0] + n))
            else:
                assert np.array_equal(blocks, np.sort(np.flatnonzero(free))[:n])
            held[k] = blocks
        st = nat.stats()
        assert st["evictions"] == ref.evictions
        assert st["used_blocks"] == ref.used == sum(ref.entries.values())
        assert st["entries"] == len(ref.entries)
        for k in range(nkeys):
            assert nat.contains(k) == (k in ref.entries)
    finally:
        nat.close()


def test_native_cache_errors():
    c = BlockCache(8)
    try:
        assert c.access(7, 3)[0] is False
        with pytest.raises(Exception):
            c.access(7, 4)                               # cached with another size
        assert c.access(9, 9) == (False, None)           # larger than the cache
        st = c.stats()
        assert st["misses"] == 2 and st["entries"] == 1 and st["free_extents"] == 1
    finally:
        c.close()
    with pytest.raises(Exception):
        BlockCache(0)


# ----------------------------------------------------------------------------- simulator
@pytest.mark.parametrize("policy", cache_sim.POLICIES)
@pytest.mark.parametrize("cap", [150, 1200])
def test_simulator_matches_reference(policy, cap):
    lens, reqs = cache_stream(11, n_docs=300, doc_len=(16, 400), docs_per_req=5, alpha=1.1, n_requests=800)
    got = cache_sim.simulate(policy, lens, reqs, cap)
    ref = ref_simulate(policy, lens, reqs, cap)
    assert (got["hit_blocks"], got["miss_blocks"]) == (ref["hit_blocks"], ref["miss_blocks"])
    if policy != "aware":        # aware's re-encoding reads are accesses the counts do not see
        assert got["evictions"] == ref["evictions"]


def test_cache_stream_shape_and_skew():
    lens, reqs = cache_stream(3, n_docs=500, docs_per_req=6, alpha=1.2, n_requests=2000)
    assert lens.shape == (500,) and reqs.shape == (2000, 6)
    assert all(len(set(r)) == 6 for r in reqs)          # distinct documents per request
    assert lens.min() >= 128 and lens.max() <= 2048
    counts = np.bincount(reqs.ravel(), minlength=500)
    top = np.sort(counts)[::-1]
    assert top[:10].sum() > 5 * top[250:260].sum()       # skewed popularity


def test_budget_sweep_rows():
    rows = cache_sim.budget_sweep(budgets_gb=(0.25, 1), n_requests=150, n_docs=300)
    assert [r["capacity_blocks"] for r in rows] == [int(g * 2 ** 30 // cache_sim.kv_bytes_per_block())
                                                  for g in (0.25, 1)]
    for r in rows:
        for p in cache_sim.POLICIES:
            assert 0.0 <= r[f"hit_ratio_{p}"] <= 1.0
        # one copy per document never loses to keying copies by offset or by sequence here
        assert r["hit_ratio_agnostic"] >= max(r["hit_ratio_aware"], r["hit_ratio_aware_exact"], r["hit_ratio_prefix"])


def test_cache_capacity_is_bounded_by_the_block_id_field():
    # block ids are 17 bits in the table word, so a cache over more blocks cannot be addressed
    c = BlockCache(1 << 17)
    try:
        hit, blocks = c.access(1, 5)
        assert not hit and blocks.tolist() == [0, 1, 2, 3, 4]
    finally:
        c.close()
    with pytest.raises(Exception):
        BlockCache((1 << 17) + 1)


def test_cache_stream_rank_order():
    lens, ranked = cache_stream(3, n_docs=500, docs_per_req=6, alpha=1.2, n_requests=1500, order="rank")
    counts = np.bincount(ranked.ravel(), minlength=500)
    top = int(np.argmax(counts))
    # the most popular document, whenever drawn, comes first
    rows = np.flatnonzero((ranked == top).any(axis=1))
    assert rows.size > 100 and np.all(ranked[rows, 0] == top)
    with pytest.raises(ValueError):
        cache_stream(3, n_requests=2, order="sorted")


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=60, deadline=None)
@given(cap=st.integers(1, 40),
       ops=st.lists(st.tuples(st.integers(0, 15), st.integers(1, 45)), min_size=1, max_size=120))
def test_native_cache_matches_reference_on_arbitrary_sequences(cap, ops):
    """Any sequence of (key, size) uses: the same hits as the reference LRU, and after every use
    the cached entries' blocks are disjoint, in range and add up to the blocks in use."""
    sizes = {}
    ref, nat, held = RefLRU(cap), BlockCache(cap), {}
    try:
        for key, n in ops:
            n = sizes.setdefault(key, n)            # an entry keeps its size
            want = ref.access(key, n)
            got, blocks = nat.access(key, n)
            assert got is want
            if blocks is not None:
                held[key] = blocks
            live = [held[k] for k in ref.entries]
            allb = np.concatenate(live) if live else np.zeros(0, np.int32)
            assert len(set(allb.tolist())) == allb.size == ref.used
            assert allb.size == 0 or (allb.min() >= 0 and allb.max() < cap)
        st_ = nat.stats()
        assert st_["used_blocks"] == ref.used and st_["entries"] == len(ref.entries)
        assert st_["evictions"] == ref.evictions
    finally:
        nat.close()
