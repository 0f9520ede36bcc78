"""GPU parity: split-KV sparse decode and anchor top-k against the fp64 oracle.

Index sets must be bit-exact (inputs carry an enforced score gap at the k-th
boundary); attention outputs must be within 2e-2 max-abs and 1e-2 mean-abs.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_aware_b200 as sa
from sparse_attention_aware_b200 import workloads as W
from tests.helpers import assert_close_attn, dense_kv, enforce_gap, head_gap_ok

pytestmark = pytest.mark.gpu


def _gpu_cache(cache, dev):
    return cache.to(dev)


def _random_idx(seed, B, Hq, kcap, lens, counts):
    rng = np.random.default_rng(seed)
    idx = np.full((B, Hq, kcap), -1, dtype=np.int32)
    cnt = np.zeros((B, Hq), dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            n = min(counts[(b * Hq + h) % len(counts)], lens[b], kcap)
            idx[b, h, :n] = np.sort(rng.choice(lens[b], n, replace=False))
            cnt[b, h] = n
    return idx, cnt


@pytest.mark.parametrize("d,P,qdt,Hq,Hkv,splits", [
    (128, 16, torch.bfloat16, 8, 2, 1),
    (128, 16, torch.bfloat16, 8, 2, 3),
    (128, 64, torch.bfloat16, 4, 4, 8),
    (64, 16, torch.float32, 4, 4, 2),
    (64, 64, torch.bfloat16, 6, 2, 5),
    (128, 16, torch.float32, 16, 2, 64),
])
def test_decode_tokens_random(cuda_dev, d, P, qdt, Hq, Hkv, splits):
    lens = [1, 37, 300, 1029]
    B = len(lens)
    cache, q = W.random_decode(11 + d + P + splits, B, Hq, Hkv, d, lens, P, q_dtype=qdt)
    kcap = 700
    idx, cnt = _random_idx(5, B, Hq, kcap, lens, [0, 1, 2, 17, 256, 700])
    scale = 1 / math.sqrt(d)
    ref, ref_lse = oracle.decode_tokens(cache, q, idx, cnt, scale)
    gc = cache.to(cuda_dev)
    sel = sa.TokenSelection(torch.from_numpy(idx).to(cuda_dev), torch.from_numpy(cnt).to(cuda_dev))
    ws = sa.Workspace(cuda_dev)
    out, lse = sa.sparse_decode_attn(gc, q.to(cuda_dev), sel, scale, splits, ws=ws)
    ws.raise_on_fault()
    assert_close_attn(out.float().cpu().numpy().reshape(-1, d), ref)
    lse_np = lse.cpu().numpy().reshape(-1)
    empty = cnt.reshape(-1) == 0
    assert np.all(np.isneginf(lse_np[empty])) and np.all(out.float().cpu().numpy().reshape(-1, d)[empty] == 0)
    np.testing.assert_allclose(lse_np[~empty], ref_lse[~empty], atol=2e-3, rtol=0)
    # bitwise run-to-run determinism
    out2, lse2 = sa.sparse_decode_attn(gc, q.to(cuda_dev), sel, scale, splits, ws=ws)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


@pytest.mark.parametrize("splits", [1, 2])
def test_decode_tokens_long_parts(cuda_dev, splits):
    """Parts longer than the 1024 positions a decode CTA resolves into shared
    memory at a time (up to 3000 positions in one part: three windows)."""
    lens = [5000, 2500, 3100]
    cache, q = W.random_decode(23 + splits, len(lens), 8, 2, 128, lens, 16)
    idx, cnt = _random_idx(9 + splits, len(lens), 8, 3000, lens, [3000, 2047, 1025, 1])
    scale = 1 / math.sqrt(128)
    ref, ref_lse = oracle.decode_tokens(cache, q, idx, cnt, scale)
    gc = cache.to(cuda_dev)
    sel = sa.TokenSelection(torch.from_numpy(idx).to(cuda_dev), torch.from_numpy(cnt).to(cuda_dev))
    ws = sa.Workspace(cuda_dev)
    out, lse = sa.sparse_decode_attn(gc, q.to(cuda_dev), sel, scale, splits, ws=ws)
    ws.raise_on_fault()
    assert_close_attn(out.float().cpu().numpy().reshape(-1, 128), ref)
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1), ref_lse, atol=2e-3, rtol=0)


def test_decode_split_invariance(cuda_dev):
    cache, q = W.random_decode(3, 2, 8, 2, 128, [2000, 999], 16)
    idx, cnt = _random_idx(1, 2, 8, 1024, [2000, 999], [1024, 900, 33])
    gc = cache.to(cuda_dev)
    sel = sa.TokenSelection(torch.from_numpy(idx).to(cuda_dev), torch.from_numpy(cnt).to(cuda_dev))
    outs = [sa.sparse_decode_attn(gc, q.to(cuda_dev), sel, 0.1, s)[0].float() for s in (1, 2, 7, 32)]
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() < 1e-2


def test_bad_device_data_is_recorded_not_faulted(cuda_dev):
    cache, q = W.random_decode(4, 2, 4, 2, 128, [100, 64], 16)
    idx, cnt = _random_idx(2, 2, 4, 32, [100, 64], [32])
    pt = cache.page_table.clone()
    pt[0, 2] = 10 ** 6                      # out-of-range physical page
    bad = W.PagedCache(cache.k, cache.v, pt, cache.seq_lens).to(cuda_dev)
    idx_bad = idx.copy()
    idx_bad[1, 0, 0] = 5000                 # index beyond the sequence
    sel = sa.TokenSelection(torch.from_numpy(idx_bad).to(cuda_dev), torch.from_numpy(cnt).to(cuda_dev))
    ws = sa.Workspace(cuda_dev)
    out, _ = sa.sparse_decode_attn(bad, q.to(cuda_dev), sel, 0.1, 2, ws=ws)
    st, det = ws.status()
    assert st == 5 and det[1] in (2, 3)      # SA_ERR_DEVICE_FAULT: page or index check
    assert ws.status()[0] == 0               # cleared after reading
    assert torch.isfinite(out.float()).all()


# --------------------------------------------------------------------------
# top-k
# --------------------------------------------------------------------------
@pytest.mark.parametrize("d,P,Hq,Hkv,k,qdt", [
    (128, 16, 8, 2, 64, torch.bfloat16),
    (128, 64, 8, 1, 100, torch.bfloat16),
    (64, 16, 4, 4, 33, torch.float32),
    (128, 16, 16, 2, 512, torch.bfloat16),
    # 8 query heads per kv head (two compute steps per ring tile), one query
    # head per kv head (256-token tiles of four 64-token pages)
    (128, 16, 8, 1, 50, torch.bfloat16),
    (64, 64, 8, 1, 40, torch.float32),
    (128, 64, 2, 2, 70, torch.bfloat16),
])
def test_topk_bit_exact_random(cuda_dev, d, P, Hq, Hkv, k, qdt):
    lens = [5, k, k + 1, 3000, 4100]
    B = len(lens)
    seed = 40 + d + k
    cache, q = W.random_decode(seed, B, Hq, Hkv, d, lens, P, q_dtype=qdt)
    q, _ = enforce_gap(cache, q, k, seed)
    ref_idx, ref_cnt = oracle.select_topk(cache, q, k)
    ws = sa.Workspace(cuda_dev)
    sel = sa.select_topk(cache.to(cuda_dev), q.to(cuda_dev), k, ws=ws)
    ws.raise_on_fault()
    np.testing.assert_array_equal(sel.count.cpu().numpy(), ref_cnt)
    np.testing.assert_array_equal(sel.idx.cpu().numpy(), ref_idx)


def test_topk_bad_page_is_recorded_and_never_selected(cuda_dev):
    cache, q = W.random_decode(8, 2, 4, 2, 128, [300, 200], 16)
    pt = cache.page_table.clone()
    pt[0, 2] = 10 ** 6                      # tokens 32..47 of sequence 0
    bad = W.PagedCache(cache.k, cache.v, pt, cache.seq_lens).to(cuda_dev)
    ws = sa.Workspace(cuda_dev)
    sel = sa.select_topk(bad, q.to(cuda_dev), 40, ws=ws)
    st, det = ws.status()
    assert st == 5 and det[1] == 2           # SA_ERR_DEVICE_FAULT, page check
    idx = sel.idx.cpu().numpy()
    assert (sel.count.cpu().numpy() == 40).all()
    assert not np.isin(idx[0], np.arange(32, 48)).any()


def test_topk_ties_go_to_lower_position(cuda_dev):
    cache, q = W.random_decode(6, 1, 2, 1, 128, [3000], 16, shuffle=True)
    k = cache.k.clone()
    k[:] = k[0, 0, 0]
    cache = W.PagedCache(k, cache.v, cache.page_table, cache.seq_lens)
    sel = sa.select_topk(cache.to(cuda_dev), q.to(cuda_dev), 77)
    assert sel.idx.cpu().tolist() == [[list(range(77))] * 2]


# --------------------------------------------------------------------------
# Tiny decode: anchor top-k over 4096 tokens + 2 reuse layers (fp32 Q)
# --------------------------------------------------------------------------
def _tiny_with_gap():
    """Tiny decode with each head's anchor query redrawn (and its planted keys
    re-aimed) until the top-k boundary gap holds."""
    subs = [0, 0, 0, 0]
    for attempt in range(200):
        wl = W.tiny_decode(1001, q_subseed=subs)
        ok = True
        for h in range(4):
            K, _ = dense_kv(wl.cache, 0, h, 4096)
            if not head_gap_ok(K.numpy(), K.abs().numpy(), wl.q_layers[0][0, h].double().numpy(), wl.k):
                subs[h] += 1
                ok = False
        if ok:
            return wl
    raise RuntimeError("no gap")


def test_tiny_decode_anchor_and_reuse(cuda_dev):
    wl = _tiny_with_gap()
    ref_idx, ref_cnt = oracle.select_topk(wl.cache, wl.q_layers[0], wl.k)
    gc = wl.cache.to(cuda_dev)
    ws = sa.Workspace(cuda_dev)
    sel = sa.select_topk(gc, wl.q_layers[0].to(cuda_dev), wl.k, ws=ws)
    np.testing.assert_array_equal(sel.idx.cpu().numpy(), ref_idx)
    for h in range(4):
        assert set(wl.planted[0, h].tolist()) <= set(sel.idx[0, h].cpu().tolist())
    scale = 1 / 8.0
    for li in range(3):
        v = wl.v_layers[li]
        ref, _ = oracle.decode_tokens(wl.cache, wl.q_layers[li], ref_idx, ref_cnt, scale, v=v)
        out, _ = sa.sparse_decode_attn(gc.with_v(v.to(cuda_dev)), wl.q_layers[li].to(cuda_dev), sel, scale, 1,
                                       ws=ws)
        assert_close_attn(out.float().cpu().numpy().reshape(-1, 64), ref)
    ws.raise_on_fault()


# --------------------------------------------------------------------------
# GQA decode at full size: B=8, 32/8 heads, d=128, L=32768, 16-token shuffled
# pages, top-k 2048 per query head, anchor + 3 reuse layers, 8 splits
# --------------------------------------------------------------------------
def test_gqa_decode_full_size(cuda_dev):
    wl = W.gqa_decode(1002)
    q0, n = enforce_gap(wl.cache, wl.q_layers[0], wl.k, 1002)
    wl.q_layers[0] = q0
    ref_idx, ref_cnt = oracle.select_topk(wl.cache, q0, wl.k)
    gc = wl.cache.to(cuda_dev)
    ws = sa.Workspace(cuda_dev)
    sel = sa.select_topk(gc, q0.to(cuda_dev), wl.k, ws=ws)
    np.testing.assert_array_equal(sel.count.cpu().numpy(), ref_cnt)
    np.testing.assert_array_equal(sel.idx.cpu().numpy(), ref_idx)
    scale = 1 / math.sqrt(128)
    for li in range(4):
        v = wl.v_layers[li]
        ref, ref_lse = oracle.decode_tokens(wl.cache, wl.q_layers[li], ref_idx, ref_cnt, scale, v=v)
        out, lse = sa.sparse_decode_attn(gc.with_v(v.to(cuda_dev)), wl.q_layers[li].to(cuda_dev), sel, scale,
                                         wl.num_splits, ws=ws)
        assert_close_attn(out.float().cpu().numpy().reshape(-1, 128), ref)
        np.testing.assert_allclose(lse.cpu().numpy().reshape(-1), ref_lse, atol=2e-3, rtol=0)
    ws.raise_on_fault()


# --------------------------------------------------------------------------
# The bench's decode configuration, in the bench's launch configuration:
# B=32, 32/8 heads, d=128, L=65536, 16-token shuffled pages, top-k 4096 per
# query head, 8 splits.  Top-k bit-exact on every row; the anchor layer and a
# reuse layer checked on sampled rows.
# --------------------------------------------------------------------------
def test_bench_decode_config(cuda_dev):
    wl = W.gqa_decode(1005, device=cuda_dev, B=32, Hq=32, Hkv=8, d=128, L=65536, P=16, k=4096, layers=2,
                      num_splits=8)
    cpu = wl.cache.to("cpu")
    q0, _ = enforce_gap(cpu, wl.q_layers[0].cpu(), wl.k, 1005)
    ref_idx, ref_cnt = oracle.select_topk(cpu, q0, wl.k)
    ws = sa.Workspace(cuda_dev)
    sel = sa.select_topk(wl.cache, q0.to(cuda_dev), wl.k, ws=ws)
    np.testing.assert_array_equal(sel.count.cpu().numpy(), ref_cnt)
    np.testing.assert_array_equal(sel.idx.cpu().numpy(), ref_idx)
    rows = np.random.default_rng(11).choice(32 * 32, 64, replace=False)
    scale = 1 / math.sqrt(128)
    for li, q in enumerate([q0, wl.q_layers[1].cpu()]):
        v = wl.v_layers[li]
        ref, ref_lse = oracle.decode_tokens(cpu, q, ref_idx, ref_cnt, scale, v=v.cpu(), rows=rows)
        out, lse = sa.sparse_decode_attn(wl.cache.with_v(v), q.to(cuda_dev), sel, scale, wl.num_splits, ws=ws)
        assert_close_attn(out.float().cpu().numpy().reshape(-1, 128)[rows], ref)
        np.testing.assert_allclose(lse.cpu().numpy().reshape(-1)[rows], ref_lse, atol=2e-3, rtol=0)
    ws.raise_on_fault()


def test_default_workspaces_are_per_stream(cuda_dev):
    """Calls without an explicit workspace on two streams get separate default
    workspaces, so decodes queued on both streams at once do not share
    split-KV scratch: each equals the same decode run alone."""
    import sparse_attention_aware_b200.api as api
    cache, q = W.random_decode(31, 4, 16, 4, 128, [3000, 1777, 4096, 900], 16)
    gc, qd = cache.to(cuda_dev), q.to(cuda_dev)
    rng = np.random.default_rng(31)
    sels = []
    for seed in (1, 2):
        idx = np.full((4, 16, 512), -1, dtype=np.int32)
        cnt = np.zeros((4, 16), dtype=np.int32)
        for b, L in enumerate([3000, 1777, 4096, 900]):
            for h in range(16):
                n = int(rng.integers(1, 512))
                idx[b, h, :n] = np.sort(rng.choice(L, n, replace=False))
                cnt[b, h] = n
        sels.append(sa.TokenSelection(torch.from_numpy(idx).to(cuda_dev), torch.from_numpy(cnt).to(cuda_dev)))
    want = [sa.sparse_decode_attn(gc, qd, s, 0.09, 8, ws=sa.Workspace(cuda_dev))[0] for s in sels]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(cuda_dev), torch.cuda.Stream(cuda_dev)]
    got = [None, None]
    for rep in range(3):
        for i, s in enumerate(streams):
            got[i] = sa.sparse_decode_attn(gc, qd, sels[i], 0.09, 8, stream=s)[0]
        torch.cuda.synchronize()
        for i in range(2):
            assert torch.equal(got[i], want[i])
    keys = [k for k in api._default_ws if k[0] == str(cuda_dev)]
    assert {k[1] for k in keys} >= {int(s.cuda_stream) for s in streams}
