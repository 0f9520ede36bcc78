"""Tiered KV host bookkeeping (CPU): residency, LRU eviction, pages of the
step in flight never evicted, capacity errors, span -> page sets."""
import numpy as np
import pytest

from sparse_attention_aware_b200 import tiered as T


def test_hits_misses_and_lru_eviction():
    m = T.SlotMap(100, 3)
    assert m.plan([5, 6]) == [(5, 0), (6, 1)]
    assert m.plan([6, 7]) == [(7, 2)]                     # 6 hits, 7 takes the free slot
    assert m.plan([8], in_flight=set()) == [(8, 0)]       # LRU: page 5 (slot 0, last used step 1)
    assert m.plan([9], in_flight=set()) == [(9, 1)]       # pages 6 and 7 were last used together: lower slot first
    assert m.stats == {"hits": 1, "misses": 5}
    assert sorted(int(p) for p in m.page_in) == [7, 8, 9]
    for s, p in enumerate(m.page_in):
        assert m.slot_of[p] == s


def test_pages_of_the_step_in_flight_are_kept():
    m = T.SlotMap(50, 4)
    m.plan([1, 2])
    m.plan([3, 4])
    pairs = m.plan([5, 6])               # the previous plan's pages {3, 4} are in flight: evict 1 and 2
    assert sorted(p for p, _ in pairs) == [5, 6]
    assert set(int(p) for p in m.page_in) == {3, 4, 5, 6}
    with pytest.raises(RuntimeError):
        m.plan([7, 8, 9])                # 5 and 6 are in flight, only the slots of 3 and 4 can be reused

def test_capacity_errors():
    m = T.SlotMap(20, 2)
    with pytest.raises(RuntimeError):
        m.plan([1, 2, 3])
    m.plan([1, 2])
    with pytest.raises(RuntimeError):
        m.plan([3, 4])                   # both slots hold the step in flight


def test_duplicates_and_repeat_hits():
    m = T.SlotMap(10, 2)
    assert m.plan([3, 3, 4, 3]) == [(3, 0), (4, 1)]
    assert m.plan([4, 3]) == []
    assert m.stats["hits"] == 2


def test_span_pages():
    assert T.span_pages([(0, 4, False), (5000, 6024, False)], 6000, 16) == [0] + list(range(312, 375))
    assert T.span_pages([(-100, 20, True), (15, 33, True)], 30, 16) == [0, 1]
    assert T.span_pages([(40, 40, True), (90, 120, True)], 64, 16) == []


def _reference_plan(state, wanted, keep):
    """The planning rule written out with numpy (test reference): distinct
    wanted pages in first-occurrence order; hits refresh their slot's tick;
    missing pages take free slots (ascending), then the least recently used
    slots (ties to the lower slot) whose page is neither wanted nor kept."""
    slot_of, page_in, last_use, tick = state
    w = np.asarray(wanted, dtype=np.int64)
    _, first = np.unique(w, return_index=True)
    w = w[np.sort(first)]
    if len(w) > len(page_in):
        return None
    keep_all = np.union1d(w, np.asarray(keep, dtype=np.int64))
    sl = slot_of[w]
    missing = w[sl < 0]
    free = np.nonzero(page_in < 0)[0]
    cand = free
    if len(free) < len(missing):
        used = np.nonzero((page_in >= 0) & ~np.isin(page_in, keep_all))[0]
        used = used[np.lexsort((used, last_use[used]))]
        cand = np.concatenate([free, used[: len(missing) - len(free)]])
    if len(cand) < len(missing):
        return None
    last_use[sl[sl >= 0]] = tick
    cand = cand[: len(missing)]
    old = page_in[cand]
    ev = old[old >= 0]
    slot_of[ev] = -1
    page_in[cand] = missing
    slot_of[missing] = cand
    last_use[cand] = tick
    return list(zip(missing.tolist(), cand.tolist())), ev.tolist(), int((sl >= 0).sum())


def test_native_plan_matches_the_rule_on_random_streams():
    rng = np.random.default_rng(7)
    for trial in range(20):
        host_pages, slots = int(rng.integers(20, 400)), int(rng.integers(4, 64))
        m = T.SlotMap(host_pages, slots)
        ref = (np.full(host_pages, -1, np.int64), np.full(slots, -1, np.int64), np.full(slots, -1, np.int64), 0)
        prev = []
        for step in range(40):
            n = int(rng.integers(0, slots + 3))
            base = int(rng.integers(0, host_pages))
            wanted = ((base + rng.integers(0, max(1, 2 * slots), n)) % host_pages).tolist()
            inflight = None if rng.random() < 0.7 else set(rng.integers(0, host_pages, 3).tolist())
            keep = prev if inflight is None else sorted(inflight)
            tick = step + 1
            ref_state = (ref[0], ref[1], ref[2], tick)
            before = (ref[0].copy(), ref[1].copy(), ref[2].copy())
            want = _reference_plan(ref_state, wanted, keep)
            if want is None:
                with pytest.raises(RuntimeError):
                    m.plan(wanted, in_flight=inflight)
                ref = (before[0], before[1], before[2], tick)
                # the native call leaves the state unchanged on a capacity error
                np.testing.assert_array_equal(m.slot_of, before[0])
                np.testing.assert_array_equal(m.page_in, before[1])
                m.prev = np.asarray(prev, dtype=np.int32) if inflight is None else m.prev
                continue
            pairs, ev, hits = want
            hits0 = m.stats["hits"]
            assert m.plan(wanted, in_flight=inflight) == pairs
            assert m.evicted == ev and m.stats["hits"] - hits0 == hits
            np.testing.assert_array_equal(m.slot_of, ref[0])
            np.testing.assert_array_equal(m.page_in, ref[1])
            np.testing.assert_array_equal(m.last_use, ref[2])
            prev = wanted


def test_native_plan_rejects_bad_pages():
    m = T.SlotMap(10, 2)
    with pytest.raises(ValueError):
        m.plan([10])
    with pytest.raises(ValueError):
        m.plan([-1])


def test_span_pages_matches_the_set_definition():
    rng = np.random.default_rng(3)
    for _ in range(200):
        L, P = int(rng.integers(1, 5000)), int(rng.choice([16, 64]))
        spans = [(int(a), int(a + rng.integers(-50, 900)), bool(rng.integers(0, 2)))
                 for a in rng.integers(-100, L + 100, int(rng.integers(0, 4)))]
        want = sorted({t // P for a, b, _ in spans for t in range(max(a, 0), min(b, L))})
        assert T.span_pages(spans, L, P) == want


def test_tier_plan_abi_scratch_and_errors():
    """The C entry point directly: the scratch size formula, a short scratch
    (SA_ERR_WORKSPACE), too many distinct pages (SA_ERR_CAPACITY) with the
    state left unchanged, and a first call on a zero-filled scratch."""
    from sparse_attention_aware_b200 import _lib
    lib = _lib.load()
    hp, slots = 50, 3
    need = lib.sa_tier_plan_scratch_ints(hp, slots)
    assert need == 1 + hp + 4 * slots and lib.sa_tier_plan_scratch_ints(0, slots) == 0
    slot_of = np.full(hp, -1, np.int32)
    page_in = np.full(slots, -1, np.int32)
    last_use = np.full(slots, -1, np.int64)
    pairs = np.zeros((slots, 2), np.int32)
    ev = np.zeros(slots, np.int32)
    counts = np.zeros(4, np.int32)
    scratch = np.zeros(need, np.int32)

    def call(wanted, scr=scratch, n_scr=None):
        w = np.asarray(wanted, np.int32)
        return lib.sa_tier_plan(slot_of.ctypes.data, hp, page_in.ctypes.data, last_use.ctypes.data, slots, 1,
                                w.ctypes.data, len(w), None, 0, pairs.ctypes.data, ev.ctypes.data,
                                counts.ctypes.data, scr.ctypes.data, need if n_scr is None else n_scr)

    assert call([1], n_scr=need - 1) == 3                    # SA_ERR_WORKSPACE
    assert call([1, 2, 3, 4]) == 7                          # SA_ERR_CAPACITY: 4 distinct > 3 slots
    assert (slot_of == -1).all() and (page_in == -1).all()
    assert call([4, 4, 9]) == 0
    assert counts.tolist() == [2, 0, 0, 2] and pairs[:2].tolist() == [[4, 0], [9, 1]]
    assert call([9, 4, 7, 9]) == 0 and counts.tolist() == [1, 0, 2, 3] and pairs[0].tolist() == [7, 2]
