"""GPU parity: causal block-sparse prefill (tcgen05) against the fp64 oracle.

Outputs within 2e-2 max-abs / 1e-2 mean-abs; LSE within 2e-3.  Masks: full
causal, diagonal only, random CSR (with empty rows), and RBS-selected; token
counts that leave a partial last block and an odd number of query blocks.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_aware_b200 as sa
from sparse_attention_aware_b200 import workloads as W
from tests.helpers import assert_close_attn, csr_to_mask, tau_in_gap

pytestmark = pytest.mark.gpu


def _mask_to_csr(mask, Hq, nB, dev):
    rows, cols = [0], []
    for h in range(Hq):
        for i in range(nB):
            sel = np.nonzero(mask[h, i * (i + 1) // 2: i * (i + 1) // 2 + i + 1])[0]
            cols.extend(sel.tolist())
            rows.append(len(cols))
    rp = torch.tensor(rows, dtype=torch.int32, device=dev)
    cl = torch.tensor(cols or [0], dtype=torch.int32, device=dev)
    return sa.BlockCSR(rp, cl, torch.zeros((2, Hq), device=dev), Hq, nB)


def _random_mask(seed, Hq, nB, density, empty_rows=0):
    rng = np.random.default_rng(seed)
    nP = nB * (nB + 1) // 2
    m = (rng.random((Hq, nP)) < density).astype(np.uint8)
    for h in range(Hq):
        for i in range(nB):
            if rng.random() < 0.5:
                m[h, i * (i + 1) // 2 + i] = 1
    for e in range(empty_rows):
        h, i = int(rng.integers(Hq)), int(rng.integers(nB))
        m[h, i * (i + 1) // 2: i * (i + 1) // 2 + i + 1] = 0
    return m


def _run(cuda_dev, wl, mask, rows=None):
    T, Hq, d = wl.q.shape
    nB = (T + 63) // 64
    scale = 1 / math.sqrt(d)
    csr = _mask_to_csr(mask, Hq, nB, cuda_dev)
    ws = sa.Workspace(cuda_dev)
    out, lse = sa.sparse_prefill_attn(wl.cache.to(cuda_dev), wl.q.to(cuda_dev), csr, scale, ws=ws)
    ws.raise_on_fault()
    ref, ref_lse = oracle.prefill(wl.cache, wl.q, 64, mask, scale, rows=rows)
    g_out = out.float().cpu().numpy().reshape(-1, d)
    g_lse = lse.cpu().numpy().reshape(-1)
    if rows is not None:
        g_out, g_lse = g_out[rows], g_lse[rows]
    assert_close_attn(g_out, ref)
    fin = np.isfinite(ref_lse)
    assert np.all(np.isneginf(g_lse[~fin])) and np.all(g_out[~fin] == 0)
    np.testing.assert_allclose(g_lse[fin], ref_lse[fin], atol=2e-3, rtol=0)
    return out, lse


@pytest.mark.parametrize("T,Hq,Hkv", [(640, 4, 2), (1000, 4, 4), (130, 2, 1), (64, 1, 1), (200, 8, 2)])
def test_prefill_full_causal(cuda_dev, T, Hq, Hkv):
    wl = W.random_prefill(300 + T, T, Hq, Hkv, 128, 64)
    nB = (T + 63) // 64
    _run(cuda_dev, wl, np.ones((Hq, nB * (nB + 1) // 2), dtype=np.uint8))


@pytest.mark.parametrize("T", [640, 777])
def test_prefill_diagonal_only_and_random(cuda_dev, T):
    Hq, Hkv = 4, 2
    wl = W.random_prefill(400 + T, T, Hq, Hkv, 128, 64)
    nB = (T + 63) // 64
    nP = nB * (nB + 1) // 2
    diag = np.zeros((Hq, nP), dtype=np.uint8)
    for i in range(nB):
        diag[:, i * (i + 1) // 2 + i] = 1
    _run(cuda_dev, wl, diag)
    _run(cuda_dev, wl, _random_mask(T, Hq, nB, 0.3, empty_rows=3))


def test_prefill_clustered_rbs_selection(cuda_dev):
    """RBS-selected masks on clustered keys with outliers (large score range)."""
    T, Hq, Hkv = 2048 + 64 * 3 + 17, 8, 2
    wl = W.clustered_prefill(501, T=T, Hq=Hq, Hkv=Hkv, d=128, block=64, n_clusters=32)
    scale = 1 / math.sqrt(128)
    c, r = oracle.block_stats(wl.cache, 64)
    qbar, qn = oracle.pool_q(wl.q, 64)
    Sc, Sr = oracle.pair_scores(qbar, qn, c, r, scale)
    tc = [tau_in_gap(Sc[h], 0.9)[0] for h in range(Hq)]
    tr = [tau_in_gap(Sr[h], 0.93)[0] for h in range(Hq)]
    mask = oracle.rbs_mask(Sc, Sr, tc, tr, True, True)
    ws = sa.Workspace(cuda_dev)
    gc = wl.cache.to(cuda_dev)
    csr = sa.select_blocks_rbs(gc, wl.q.to(cuda_dev), 64, scale, tau_c=torch.tensor(tc), tau_r=torch.tensor(tr),
                               ws=ws)
    nB = (T + 63) // 64
    rp = csr.row_ptr.cpu().numpy()
    np.testing.assert_array_equal(csr_to_mask(rp, csr.cols.cpu().numpy()[: rp[-1]], Hq, nB), mask)
    out, lse = sa.sparse_prefill_attn(gc, wl.q.to(cuda_dev), csr, scale, ws=ws)
    ws.raise_on_fault()
    ref, _ = oracle.prefill(wl.cache, wl.q, 64, mask, scale)
    assert_close_attn(out.float().cpu().numpy().reshape(-1, 128), ref)
    out2, lse2 = sa.sparse_prefill_attn(gc, wl.q.to(cuda_dev), csr, scale, ws=ws)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_prefill_block_sparse_full_size_sampled(cuda_dev):
    """32768 tokens, 32/4 heads, RBS-selected blocks; sampled query rows."""
    wl = W.clustered_prefill(1004)
    T, Hq, d = wl.q.shape
    scale = 1 / math.sqrt(128)
    c, r = oracle.block_stats(wl.cache, 64)
    qbar, qn = oracle.pool_q(wl.q, 64)
    Sc, Sr = oracle.pair_scores(qbar, qn, c, r, scale)
    tc = [tau_in_gap(Sc[h], 0.95)[0] for h in range(Hq)]
    tr = [tau_in_gap(Sr[h], 0.97)[0] for h in range(Hq)]
    mask = oracle.rbs_mask(Sc, Sr, tc, tr, True, True)
    rng = np.random.default_rng(5)
    ts = np.concatenate([[0, 63, 64, 127, T - 1, T - 64], rng.integers(0, T, 250)])
    hs = rng.integers(0, Hq, len(ts))
    rows = (ts * Hq + hs).astype(np.int64)
    _run(cuda_dev, wl, mask, rows=rows)


def test_bench_prefill_config(cuda_dev):
    """The bench's prefill configuration: 131072 tokens, 32/4 heads, 64x64
    blocks, clustered keys with outliers, thresholds started at the bench's
    quantile levels 0.965 / 0.985 and moved into >= 1e-3 gaps of the fp64
    scores (the fp32 pair-score error is ~1e-4; near the 96.5% quantile of
    2.1M pairs the scores lie ~1e-5 apart, so the nearest such gap sits in
    the tail and the kept density comes out near 2% rather than the bench's
    5%).  The RBS mask is compared bit for bit, the prefill output on
    sampled rows."""
    wl = W.clustered_prefill(1005, device=cuda_dev, T=131072, Hq=32, Hkv=4, d=128, block=64)
    T, Hq, d = wl.q.shape
    scale = 1 / math.sqrt(128)
    cpu = wl.cache.to("cpu")
    qc = wl.q.cpu()
    c, r = oracle.block_stats(cpu, 64)
    qbar, qn = oracle.pool_q(qc, 64)
    Sc, Sr = oracle.pair_scores(qbar, qn, c, r, scale)
    tc = [tau_in_gap(Sc[h], 0.965)[0] for h in range(Hq)]
    tr = [tau_in_gap(Sr[h], 0.985)[0] for h in range(Hq)]
    mask = oracle.rbs_mask(Sc, Sr, tc, tr, True, True)
    assert 0.01 < mask.mean() < 0.08
    ws = sa.Workspace(cuda_dev)
    csr = sa.select_blocks_rbs(wl.cache, wl.q, 64, scale, tau_c=torch.tensor(tc), tau_r=torch.tensor(tr), ws=ws)
    ws.raise_on_fault()
    nB = T // 64
    got = csr_to_mask(csr.row_ptr.cpu().numpy(), csr.cols.cpu().numpy(), Hq, nB)
    np.testing.assert_array_equal(got, mask)
    out, lse = sa.sparse_prefill_attn(wl.cache, wl.q, csr, scale, ws=ws)
    ws.raise_on_fault()
    rng = np.random.default_rng(13)
    ts = np.concatenate([[0, 63, 64, T - 1, T - 64], rng.integers(0, T, 200)])
    hs = rng.integers(0, Hq, len(ts))
    rows = (ts * Hq + hs).astype(np.int64)
    ref, ref_lse = oracle.prefill(cpu, qc, 64, mask, scale, rows=rows)
    g_out = out.float().cpu().numpy().reshape(-1, d)[rows]
    assert_close_attn(g_out, ref)
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1)[rows], ref_lse, atol=2e-3, rtol=0)


def test_bench_prefill_config_at_bench_density(cuda_dev):
    """The prefill exactly as the bench times it: 131072 tokens, 32/4 heads,
    the bench's quantile levels (p_c = 0.9648, p_r = p_c + 0.02, ~5% kept
    blocks including the forced ones), per-head thresholds read back from the
    quantile-mode call and passed explicitly, and the CSR that selection
    produced executed by the tcgen05 kernel.  The oracle attends over the mask
    read back from that CSR (mask bit-exactness is the gap-threshold test's
    job) on 260 sampled rows, the first and last query blocks included."""
    wl = W.clustered_prefill(1005, device=cuda_dev, T=131072, Hq=32, Hkv=4, d=128, block=64)
    T, Hq, d = wl.q.shape
    nB = T // 64
    scale = 1 / math.sqrt(128)
    ws = sa.Workspace(cuda_dev)
    pc = 0.9648
    q_csr = sa.select_blocks_rbs(wl.cache, wl.q, 64, scale, p_c=pc, p_r=pc + 0.02, ws=ws)
    ws.raise_on_fault()
    tau = q_csr.tau.clone()
    csr = sa.select_blocks_rbs(wl.cache, wl.q, 64, scale, tau_c=tau[0], tau_r=tau[1], ws=ws)
    ws.raise_on_fault()
    mask = csr_to_mask(csr.row_ptr.cpu().numpy(), csr.cols.cpu().numpy(), Hq, nB)
    assert 0.045 <= mask.mean() <= 0.055, mask.mean()
    out, lse = sa.sparse_prefill_attn(wl.cache, wl.q, csr, scale, ws=ws)
    ws.raise_on_fault()
    rng = np.random.default_rng(29)
    ts = np.concatenate([[0, 1, 63, 64, 127, T - 64, T - 63, T - 2, T - 1],
                         rng.integers(0, 64, 8), rng.integers(T - 64, T, 8), rng.integers(0, T, 235)])
    hs = rng.integers(0, Hq, len(ts))
    rows = (ts * Hq + hs).astype(np.int64)
    cpu = wl.cache.to("cpu")
    ref, ref_lse = oracle.prefill(cpu, wl.q.cpu(), 64, mask, scale, rows=rows)
    g_out = out.float().cpu().numpy().reshape(-1, d)[rows]
    assert_close_attn(g_out, ref)
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1)[rows], ref_lse, atol=2e-3, rtol=0)


def _schedule_items(ws, Hq, Hkv, nB):
    """Work items the last prefill call left in its workspace (after the
    256-byte status header): {head A, block A, head B (-1: none), block B}."""
    G = Hq // Hkv
    n_items = (Hq // 2) * nB if (G % 2 == 0 and G <= 16) else Hq * ((nB + 1) // 2)
    buf = ws.buf
    off = (-buf.data_ptr()) % 256 + 256
    return buf[off: off + 16 * n_items].view(torch.int32).reshape(-1, 4).cpu().numpy()


@pytest.mark.parametrize("T,Hq,Hkv", [(1500, 12, 2), (1500, 16, 1), (777, 6, 2), (1300, 2, 1), (2100, 8, 1)])
def test_prefill_group_sizes_and_schedule(cuda_dev, T, Hq, Hkv):
    """Group sizes 6 and 16 (rows paired within windows of 10 and 4 query
    blocks, the last window partial), 2 and 8, and an odd group (adjacent
    query blocks of one head); random masks with empty rows.  The work items
    must cover every (head, query block) row exactly once, and the two halves
    of an item must share a kv head."""
    wl = W.random_prefill(700 + T + Hq, T, Hq, Hkv, 128, 64)
    nB = (T + 63) // 64
    mask = _random_mask(T + Hq, Hq, nB, 0.25, empty_rows=4)
    csr = _mask_to_csr(mask, Hq, nB, cuda_dev)
    ws = sa.Workspace(cuda_dev)
    scale = 1 / math.sqrt(128)
    out, lse = sa.sparse_prefill_attn(wl.cache.to(cuda_dev), wl.q.to(cuda_dev), csr, scale, ws=ws)
    ws.raise_on_fault()
    ref, ref_lse = oracle.prefill(wl.cache, wl.q, 64, mask, scale)
    g_out = out.float().cpu().numpy().reshape(-1, 128)
    g_lse = lse.cpu().numpy().reshape(-1)
    assert_close_attn(g_out, ref)
    fin = np.isfinite(ref_lse)
    assert np.all(np.isneginf(g_lse[~fin])) and np.all(g_out[~fin] == 0)
    np.testing.assert_allclose(g_lse[fin], ref_lse[fin], atol=2e-3, rtol=0)
    seen = np.zeros((Hq, nB), dtype=np.int64)
    G = Hq // Hkv
    for h0, i0, h1, i1 in _schedule_items(ws, Hq, Hkv, nB):
        assert 0 <= h0 < Hq and 0 <= i0 < nB
        seen[h0, i0] += 1
        if h1 >= 0:
            assert 0 <= h1 < Hq and 0 <= i1 < nB and h0 // G == h1 // G
            seen[h1, i1] += 1
    assert np.array_equal(seen, np.ones((Hq, nB), dtype=np.int64))


def test_prefill_longer_than_one_bitmap_chunk(cuda_dev):
    """140000 tokens (2188 query blocks): the pairing windows near the end
    build their row bitmaps in two chunks of 2048 key blocks.  Sparse random
    mask (diagonal forced), sampled rows against the oracle, and the work
    items still cover every row once."""
    T, Hq, Hkv = 140000, 2, 1
    wl = W.random_prefill(901, T, Hq, Hkv, 128, 64)
    nB = (T + 63) // 64
    rng = np.random.default_rng(17)
    nP = nB * (nB + 1) // 2
    mask = (rng.random((Hq, nP)) < 0.01).astype(np.uint8)
    for i in range(nB):
        mask[:, i * (i + 1) // 2 + i] = 1
    ts = np.concatenate([[0, 131071, 131072, 139999, T - 64], rng.integers(0, T, 120)])
    hs = rng.integers(0, Hq, len(ts))
    rows = (ts * Hq + hs).astype(np.int64)
    csr = _mask_to_csr(mask, Hq, nB, cuda_dev)
    ws = sa.Workspace(cuda_dev)
    scale = 1 / math.sqrt(128)
    out, lse = sa.sparse_prefill_attn(wl.cache.to(cuda_dev), wl.q.to(cuda_dev), csr, scale, ws=ws)
    ws.raise_on_fault()
    ref, ref_lse = oracle.prefill(wl.cache, wl.q, 64, mask, scale, rows=rows)
    assert_close_attn(out.float().cpu().numpy().reshape(-1, 128)[rows], ref)
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1)[rows], ref_lse, atol=2e-3, rtol=0)
    seen = np.zeros((Hq, nB), dtype=np.int64)
    for h0, i0, h1, i1 in _schedule_items(ws, Hq, Hkv, nB):
        seen[h0, i0] += 1
        if h1 >= 0:
            seen[h1, i1] += 1
    assert np.array_equal(seen, np.ones((Hq, nB), dtype=np.int64))
