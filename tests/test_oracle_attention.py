"""Pins for the oracle's masked softmax attention and split-KV combine (CPU).

The oracle's attention is checked against things other than itself:
torch's fp64 scaled_dot_product_attention (select-all = dense), closed forms
(constant V, a single key), a brute-force formula without max subtraction,
permutation invariance and the split/combine identity.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_aware_b200 import workloads as W
from tests.helpers import dense_kv, lse64, sdpa64


def _cache(seed=7, B=2, Hq=4, Hkv=2, d=32, lens=(37, 50), P=16):
    return W.random_decode(seed, B, Hq, Hkv, d, list(lens), P)


def _all_idx(cache, Hq, k):
    B = cache.batch
    idx = np.full((B, Hq, k), -1, dtype=np.int32)
    cnt = np.zeros((B, Hq), dtype=np.int32)
    for b in range(B):
        L = int(cache.seq_lens[b])
        idx[b, :, :L] = np.arange(L)
        cnt[b] = L
    return idx, cnt


def test_select_all_equals_dense_sdpa():
    cache, q = _cache()
    B, Hq, d = q.shape
    scale = 1 / math.sqrt(d)
    idx, cnt = _all_idx(cache, Hq, 64)
    out, lse = oracle.decode_tokens(cache, q, idx, cnt, scale)
    out = out.reshape(B, Hq, d)
    lse = lse.reshape(B, Hq)
    for b in range(B):
        L = int(cache.seq_lens[b])
        for h in range(Hq):
            K, V = dense_kv(cache, b, h // (Hq // 2), L)
            qh = q[b, h].double()[None]
            ref = sdpa64(qh, K, V, scale)[0]
            np.testing.assert_allclose(out[b, h], ref.numpy(), rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], lse64(qh, K, scale)[0].item(), rtol=0, atol=1e-12)


def test_constant_v_returns_v():
    cache, q = _cache(seed=8)
    B, Hq, d = q.shape
    const = torch.randn(d).to(torch.bfloat16)
    v = cache.v.clone()
    v[:] = const
    idx, cnt = _all_idx(cache, Hq, 64)
    out, _ = oracle.decode_tokens(cache, q, idx, cnt, 0.3, v=v)
    np.testing.assert_allclose(out, np.broadcast_to(const.double().numpy(), out.shape), rtol=0, atol=1e-12)


def test_single_key_returns_its_value():
    cache, q = _cache(seed=9)
    B, Hq, d = q.shape
    idx = np.full((B, Hq, 4), -1, dtype=np.int32)
    cnt = np.ones((B, Hq), dtype=np.int32)
    idx[:, :, 0] = 5
    out, lse = oracle.decode_tokens(cache, q, idx, cnt, 0.2)
    out, lse = out.reshape(B, Hq, d), lse.reshape(B, Hq)
    for b in range(B):
        for h in range(Hq):
            K, V = dense_kv(cache, b, h // 2, 6)
            np.testing.assert_array_equal(out[b, h], V[5].numpy())
            assert lse[b, h] == pytest.approx(0.2 * float(q[b, h].double() @ K[5]), abs=1e-12)


def test_brute_force_formula_and_permutation():
    """No max subtraction: out = sum e^s v / sum e^s; same for any order of S."""
    cache, q = _cache(seed=10, d=16)
    B, Hq, d = q.shape
    rng = np.random.default_rng(0)
    idx = np.full((B, Hq, 20), -1, dtype=np.int32)
    cnt = np.full((B, Hq), 20, dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            idx[b, h] = rng.choice(int(cache.seq_lens[b]), 20, replace=False)
    scale = 0.05
    out, lse = oracle.decode_tokens(cache, q, idx, cnt, scale)
    perm = idx[:, :, ::-1].copy()
    out2, lse2 = oracle.decode_tokens(cache, q, perm, cnt, scale)
    np.testing.assert_allclose(out, out2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-13)
    out, lse = out.reshape(B, Hq, d), lse.reshape(B, Hq)
    for b in range(B):
        for h in range(Hq):
            K, V = dense_kv(cache, b, h // 2, int(cache.seq_lens[b]))
            sel = torch.from_numpy(idx[b, h].astype(np.int64))
            e = torch.exp(scale * (K[sel] @ q[b, h].double()))
            np.testing.assert_allclose(out[b, h], ((e[:, None] * V[sel]).sum(0) / e.sum()).numpy(),
                                       rtol=0, atol=1e-12)
            assert lse[b, h] == pytest.approx(math.log(float(e.sum())), abs=1e-12)


def test_empty_set():
    cache, q = _cache(seed=11)
    B, Hq, d = q.shape
    idx = np.full((B, Hq, 4), -1, dtype=np.int32)
    cnt = np.zeros((B, Hq), dtype=np.int32)
    out, lse = oracle.decode_tokens(cache, q, idx, cnt, 0.1)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


@pytest.mark.parametrize("S", [1, 3, 8])
def test_combine_of_splits_equals_unsplit(S):
    cache, q = _cache(seed=12, lens=(37, 50))
    B, Hq, d = q.shape
    idx, cnt = _all_idx(cache, Hq, 64)
    cnt[0, 1] = 5       # fewer entries than splits -> empty splits
    out, lse, pm, pl, pa = oracle.decode_tokens_split(cache, q, idx, cnt, 0.125, S)
    for r in range(B * Hq):
        o2, l2 = oracle.combine(pm[r], pl[r], pa[r])
        np.testing.assert_allclose(o2, out[r], rtol=0, atol=1e-12)
        assert l2 == pytest.approx(lse[r], abs=1e-12)
    # all parts empty -> zeros, -inf
    o3, l3 = oracle.combine(np.full(3, -np.inf), np.zeros(3), np.zeros((3, d)))
    assert np.all(o3 == 0) and l3 == -np.inf
