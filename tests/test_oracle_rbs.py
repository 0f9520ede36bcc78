"""Pins for the oracle's RBS selection and block-sparse causal prefill (CPU).

Closed forms and invariants from the definitions: the radius bound
q.k <= q.c + ||q|| r (and its tightness), degenerate blocks (identical keys,
one token), the mean identity qbar.c = mean of the tile's q.k, numpy's
lower quantile, kept counts, and torch fp64 SDPA for the full and the
diagonal-only masks.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_aware_b200 import workloads as W
from tests.helpers import dense_kv, sdpa64


def _wl(T=200, Hq=4, Hkv=2, d=16, bs=16, seed=21, clustered=False):
    if clustered:
        return W.clustered_prefill(seed, T=T, Hq=Hq, Hkv=Hkv, d=d, block=bs, n_clusters=8,
                                   outlier_frac=0.05)
    return W.random_prefill(seed, T, Hq, Hkv, d, bs)


def _tile(wl, g, j, bs):
    K, V = dense_kv(wl.cache, 0, g, wl.T)
    return K[j * bs: min((j + 1) * bs, wl.T)]


@pytest.mark.parametrize("clustered", [False, True])
def test_radius_bound_every_key(clustered):
    wl = _wl(clustered=clustered)
    bs = wl.block
    c, r = oracle.block_stats(wl.cache, bs)
    qbar, qn = oracle.pool_q(wl.q, bs)
    Q = wl.q.double()
    nB = c.shape[1]
    for g in range(c.shape[0]):
        for j in range(nB):
            Kt = _tile(wl, g, j, bs).numpy()
            for q in [Q[j * bs % wl.T, 0].numpy(), qbar[0, j], np.random.default_rng(j).normal(size=16)]:
                lhs = Kt @ q
                rhs = q @ c[g, j] + np.linalg.norm(q) * r[g, j]
                assert np.all(lhs <= rhs + 1e-9)
            # tight: q along the farthest key's offset reaches the bound
            far = np.argmax(np.linalg.norm(Kt - c[g, j], axis=1))
            u = Kt[far] - c[g, j]
            assert np.linalg.norm(u) == pytest.approx(r[g, j], abs=1e-12)
            if r[g, j] > 0:
                assert Kt[far] @ u == pytest.approx(u @ c[g, j] + np.linalg.norm(u) * r[g, j], rel=1e-12)


def test_degenerate_blocks():
    wl = _wl(T=40, bs=16, seed=22)
    k = wl.cache.k.clone()
    pt = wl.cache.page_table[0].long()
    k[pt[0]] = k[pt[0], :, :1]            # block 0: 16 identical keys
    cache = W.PagedCache(k, wl.cache.v, wl.cache.page_table, wl.cache.seq_lens)
    c, r = oracle.block_stats(cache, 16)
    K, _ = dense_kv(cache, 0, 1, 40)
    assert r[1, 0] == 0.0 and np.array_equal(c[1, 0], K[0].numpy())
    # T = 40, bs = 16 -> block 2 holds 8 tokens; bs = 1 -> every block one token
    c1, r1 = oracle.block_stats(cache, 1)
    assert np.all(r1 == 0) and np.array_equal(c1[1], K.numpy())
    qbar, qn = oracle.pool_q(wl.q, 16)
    Sc, Sr = oracle.pair_scores(qbar, qn, c, r, 0.5)
    for i in range(3):
        p = i * (i + 1) // 2 + 0
        assert Sc[2, p] == Sr[2, p]        # r = 0 -> rescue score = centroid score


def test_mean_identity_and_partial_block():
    """S_c / scale = qbar_i . c_j = mean over the tile of q.k (also for a partial last block)."""
    wl = _wl(T=70, bs=16, seed=23)
    bs, scale = 16, 0.25
    c, r = oracle.block_stats(wl.cache, bs)
    qbar, qn = oracle.pool_q(wl.q, bs)
    Sc, Sr = oracle.pair_scores(qbar, qn, c, r, scale)
    nB = 5
    Q = wl.q.double()
    for h in range(4):
        g = h // 2
        K, _ = dense_kv(wl.cache, 0, g, 70)
        for i in range(nB):
            Qi = Q[i * bs: min((i + 1) * bs, 70), h]
            for j in range(i + 1):
                Kj = K[j * bs: min((j + 1) * bs, 70)]
                p = i * (i + 1) // 2 + j
                assert Sc[h, p] == pytest.approx(scale * float((Qi @ Kj.T).mean()), abs=1e-12)
                assert Sr[h, p] == pytest.approx(Sc[h, p] + scale * qn[h, i] * r[g, j], abs=1e-12)
                assert qn[h, i] == pytest.approx(float(Qi.mean(0).norm()), abs=1e-12)


def test_quantile_matches_numpy_lower_and_kept_count():
    x = np.random.default_rng(4).normal(size=1001)
    for p in [0.0, 0.3, 0.95, 0.97, 1.0]:
        tau = oracle.quantile(x, p)
        assert tau == np.quantile(x, p, method="lower")
        assert int((x > tau).sum()) == len(x) - 1 - math.floor(p * (len(x) - 1))
    assert np.array_equal(oracle.sort(x), np.sort(x))


def test_mask_structure():
    wl = _wl(T=256, bs=16, seed=24, clustered=True)
    c, r = oracle.block_stats(wl.cache, 16)
    qbar, qn = oracle.pool_q(wl.q, 16)
    Sc, Sr = oracle.pair_scores(qbar, qn, c, r, 0.25)
    nB = 16
    tc = [oracle.quantile(Sc[h], 0.8) for h in range(4)]
    tr = [oracle.quantile(Sr[h], 0.9) for h in range(4)]
    m = oracle.rbs_mask(Sc, Sr, tc, tr, True, True)
    mc = oracle.rbs_mask(Sc, Sr, tc, [np.inf] * 4, False, False)
    mr = oracle.rbs_mask(Sc, Sr, [np.inf] * 4, tr, False, False)
    assert np.all(m >= mc) and np.all(m >= mr) and np.any(m > np.maximum(mc, mr))
    for h in range(4):
        assert int(mc[h].sum()) == Sc.shape[1] - 1 - math.floor(0.8 * (Sc.shape[1] - 1))
    for i in range(nB):
        assert np.all(m[:, i * (i + 1) // 2 + i] == 1) and np.all(m[:, i * (i + 1) // 2] == 1)
    full = oracle.rbs_mask(Sc, Sr, [-np.inf] * 4, [-np.inf] * 4, False, False)
    assert np.all(full == 1)
    none = oracle.rbs_mask(Sc, Sr, [np.inf] * 4, [np.inf] * 4, False, False)
    assert np.all(none == 0)


def _causal_ref(wl, h, mask_fn, scale):
    K, V = dense_kv(wl.cache, 0, h // (wl.q.shape[1] // wl.cache.num_kv_heads), wl.T)
    Q = wl.q[:, h].double()
    t = torch.arange(wl.T)
    allow = mask_fn(t[:, None], t[None, :])
    return sdpa64(Q, K, V, scale, allow)


@pytest.mark.parametrize("T,bs", [(100, 16), (64, 64), (130, 32)])
def test_prefill_full_mask_equals_dense_causal(T, bs):
    wl = _wl(T=T, bs=bs, seed=25)
    nB = (T + bs - 1) // bs
    mask = np.ones((4, nB * (nB + 1) // 2), dtype=np.uint8)
    scale = 1 / math.sqrt(16)
    out, lse = oracle.prefill(wl.cache, wl.q, bs, mask, scale)
    out = out.reshape(T, 4, 16)
    for h in range(4):
        ref = _causal_ref(wl, h, lambda a, b: b <= a, scale)
        np.testing.assert_allclose(out[:, h], ref.numpy(), rtol=0, atol=1e-12)


def test_prefill_diagonal_only_is_block_local_causal():
    T, bs = 90, 16
    wl = _wl(T=T, bs=bs, seed=26)
    c, r = oracle.block_stats(wl.cache, bs)
    qbar, qn = oracle.pool_q(wl.q, bs)
    Sc, Sr = oracle.pair_scores(qbar, qn, c, r, 0.25)
    mask = oracle.rbs_mask(Sc, Sr, [np.inf] * 4, [np.inf] * 4, True, False)
    out, _ = oracle.prefill(wl.cache, wl.q, bs, mask, 0.25)
    out = out.reshape(T, 4, 16)
    for h in range(4):
        ref = _causal_ref(wl, h, lambda a, b: (b <= a) & (a // bs == b // bs), 0.25)
        np.testing.assert_allclose(out[:, h], ref.numpy(), rtol=0, atol=1e-12)
    # a sampled-rows call agrees with the full call
    rows = [5 * 4 + 1, 77 * 4 + 3]
    o2, _ = oracle.prefill(wl.cache, wl.q, bs, mask, 0.25, rows=rows)
    np.testing.assert_array_equal(o2[0], out[5, 1])
    np.testing.assert_array_equal(o2[1], out[77, 3])
