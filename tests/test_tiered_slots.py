"""Tiered KV host bookkeeping (CPU): residency, LRU eviction, pages of the
step in flight never evicted, capacity errors, span -> page sets."""
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
