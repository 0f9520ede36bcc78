"""The prefill scheduler pairs the rows of a window greedily (repeatedly the
free pair of smallest (waste, row, row) key), computed as rounds of mutually
best pairs.  This pins the claim that the two procedures give the same
pairing under a strict order on the pairs (CPU, random and adversarial
wastes); the GPU tests check that the kernel's work items cover every row."""
import numpy as np


def _key(cost, a, b):
    lo, hi = min(a, b), max(a, b)
    return (int(cost[lo, hi]), lo, hi)


def sequential_greedy(cost, n):
    keys = sorted(_key(cost, a, b) for a in range(n) for b in range(a + 1, n))
    used, pairs = set(), set()
    for _, a, b in keys:
        if a not in used and b not in used:
            used |= {a, b}
            pairs.add((a, b))
    return pairs


def mutual_best_rounds(cost, n):
    used, pairs, rounds = set(), set(), 0
    while len(pairs) < n // 2:
        rounds += 1
        best = {}
        for a in range(n):
            if a in used:
                continue
            cands = [_key(cost, a, b) for b in range(n) if b != a and b not in used]
            if cands:
                _, lo, hi = min(cands)
                best[a] = hi if lo == a else lo
        taken = [(a, b) for a, b in best.items() if b > a and best.get(b) == a]
        assert taken, "a round must take the smallest free pair"
        for a, b in taken:
            pairs.add((a, b))
            used |= {a, b}
    return pairs, rounds


def test_rounds_equal_sequential_greedy_random():
    rng = np.random.default_rng(0)
    for trial in range(200):
        n = int(rng.choice([2, 4, 6, 10, 16, 32, 64]))
        cost = rng.integers(0, int(rng.choice([3, 20, 1000])), size=(n, n))   # many ties at small ranges
        cost = np.triu(cost, 1)
        cost = cost + cost.T
        pairs, rounds = mutual_best_rounds(cost, n)
        assert pairs == sequential_greedy(cost, n)
        assert rounds <= n // 2
        assert sorted(x for p in pairs for x in p) == list(range(n))


def test_rounds_equal_sequential_greedy_all_equal_wastes():
    # every waste equal: the order falls back to the row ids alone
    n = 64
    cost = np.zeros((n, n), dtype=np.int64)
    pairs, _ = mutual_best_rounds(cost, n)
    assert pairs == sequential_greedy(cost, n) == {(2 * i, 2 * i + 1) for i in range(n // 2)}
