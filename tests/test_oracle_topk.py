"""Pins for the oracle's anchor-layer top-k (CPU).

Brute force over every subset on tiny inputs, invariants (|S| = min(k, L),
tie-break to the lower position, head independence, positive scaling of q),
and the planted keys of the tiny-decode workload.
"""
import itertools

import numpy as np
import torch

import oracle
from sparse_attention_aware_b200 import workloads as W
from tests.helpers import dense_kv


def test_brute_force_subsets_tiny():
    rng = np.random.default_rng(3)
    for trial in range(12):
        L = int(rng.integers(2, 13))
        k = int(rng.integers(1, 5))
        cache, q = W.random_decode(100 + trial, 1, 2, 1, 8, [L], 4, q_dtype=torch.float32)
        idx, cnt = oracle.select_topk(cache, q, k)
        K, _ = dense_kv(cache, 0, 0, L)
        for h in range(2):
            r = (K @ q[0, h].double()).numpy()
            m = min(k, L)
            winners = []
            for sub in itertools.combinations(range(L), m):
                rest = [t for t in range(L) if t not in sub]
                if not rest or min(r[list(sub)]) > max(r[rest]):
                    winners.append(sub)
            assert len(winners) == 1, "scores tie at the boundary"
            assert cnt[0, h] == m
            assert list(idx[0, h, :m]) == list(winners[0])
            assert np.all(idx[0, h, m:] == -1)


def test_count_and_short_context():
    cache, q = W.random_decode(5, 3, 4, 2, 16, [3, 40, 17], 16)
    idx, cnt = oracle.select_topk(cache, q, 20)
    assert cnt.tolist() == [[3] * 4, [20] * 4, [17] * 4]
    assert list(idx[0, 0, :3]) == [0, 1, 2] and np.all(idx[0, 0, 3:] == -1)
    for b in range(3):
        for h in range(4):
            c = cnt[b, h]
            assert np.all(np.diff(idx[b, h, :c]) > 0)


def test_ties_go_to_lower_position():
    cache, q = W.random_decode(6, 1, 1, 1, 8, [32], 16, shuffle=False)
    k = cache.k.clone()
    k[:] = k[0, 0, 0]          # every key identical -> every score ties
    cache = W.PagedCache(k, cache.v, cache.page_table, cache.seq_lens)
    idx, cnt = oracle.select_topk(cache, q, 5)
    assert list(idx[0, 0]) == [0, 1, 2, 3, 4]


def test_head_independence_and_scale_invariance():
    cache, q = W.random_decode(7, 2, 8, 2, 16, [64, 50], 16)
    idx, cnt = oracle.select_topk(cache, q, 10)
    q2 = q.clone()
    q2[:, 1::2] = torch.randn_like(q2[:, 1::2].float()).to(q2.dtype)   # change the other heads
    q2[:, 0::2] = (q2[:, 0::2].float() * 4).to(q2.dtype)               # positive scale (exact in bf16)
    idx2, _ = oracle.select_topk(cache, q2, 10)
    np.testing.assert_array_equal(idx[:, 0::2], idx2[:, 0::2])


def test_tiny_decode_planted_keys_are_selected():
    wl = W.tiny_decode(1001)
    idx, cnt = oracle.select_topk(wl.cache, wl.q_layers[0], wl.k)
    assert np.all(cnt == 256)
    for h in range(4):
        planted = set(wl.planted[0, h].tolist())
        assert planted <= set(idx[0, h].tolist())
