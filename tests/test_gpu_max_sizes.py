"""Parity at the entry points' size limits (GPU).

Top-k over a 2^19-token context (the largest max_pages_per_seq * page_size
that sa_select_topk accepts) with k = 65536 (the largest k).  At this k the
select's threshold digit holds more candidates than its 4096-entry buffer,
so the full-row overflow path runs at full size.  The order statistics are
~1e-4 apart there, inside the fp32 error band of a dot product, so the check
is the definition up to that band: exactly k distinct ascending positions,
every position whose fp64 score (oracle) exceeds the k-th largest by more
than the fp32 dot-product error bound is selected, and none that falls short
of it by more than the bound.  The decode over the selected 65536 rows per
head is then compared with the oracle's decode over the same rows."""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_aware_b200 as sa
from sparse_attention_aware_b200 import workloads as W
from tests.helpers import assert_close_attn, dense_kv

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


def test_topk_and_decode_at_the_size_limits(cuda_dev):
    L, P, k, d = 1 << 19, 64, 65536, 64
    cache, q = W.random_decode(4242, 1, 2, 1, d, [L], P)
    assert cache.page_table.shape[1] * P == L          # the capacity limit itself
    gc = cache.to(cuda_dev)
    ws = sa.Workspace(cuda_dev)
    sel = sa.select_topk(gc, q.to(cuda_dev), k, ws=ws)
    ws.raise_on_fault("top-k at the size limit")
    idx, cnt = sel.idx.cpu().numpy(), sel.count.cpu().numpy()
    assert (cnt == k).all()
    r = oracle.topk_scores(cache, q)                    # fp64 [1][2][L]
    K, _ = dense_kv(cache, 0, 0, L)
    gam = (d + 1) * U32 / (1 - (d + 1) * U32)
    for h in range(2):
        sel_h = idx[0, h]
        assert np.all(np.diff(sel_h) > 0) and sel_h[0] >= 0 and sel_h[-1] < L
        s = r[0, h]
        kth = np.sort(s)[::-1][k - 1]
        band = 2 * gam * (np.abs(K.numpy()) @ np.abs(q[0, h].double().numpy()))   # per-row fp32 error bound x2
        chosen = np.zeros(L, dtype=bool)
        chosen[sel_h] = True
        assert chosen[s > kth + band].all()
        assert not chosen[s < kth - band].any()
    scale = 1 / math.sqrt(d)
    ref, ref_lse = oracle.decode_tokens(cache, q, idx, cnt, scale)
    out, lse = sa.sparse_decode_attn(gc, q.to(cuda_dev), sel, scale, 16, ws=ws)
    ws.raise_on_fault("decode at the size limit")
    assert_close_attn(out.float().cpu().numpy().reshape(-1, d), ref)
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1), ref_lse, atol=2e-3, rtol=0)


def test_topk_rejects_a_context_past_the_limit(cuda_dev):
    cache, q = W.random_decode(4243, 1, 2, 1, 64, [(1 << 19) + 64], 64)
    assert cache.page_table.shape[1] * 64 > 1 << 19
    with pytest.raises(sa.SAError):
        sa.select_topk(cache.to(cuda_dev), q.to(cuda_dev), 16)
