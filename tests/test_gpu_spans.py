"""GPU parity: span masks -> block lists (bit-exact token sets) and masked
decode over them (DA focus / local / global, LoZA streaming)."""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_aware_b200 as sa
from oracle import modes as OM
from sparse_attention_aware_b200 import spans as SP
from sparse_attention_aware_b200 import workloads as W
from tests.helpers import assert_close_attn

pytestmark = pytest.mark.gpu


def _members_from_blocks(blocks, counts, P, Lmax):
    """Token membership implied by a GPU block list; also checks every token
    appears once and entries are ascending with consistent prefix sums."""
    B = blocks.shape[0]
    mem = np.zeros((B, Lmax), dtype=np.uint8)
    for b in range(B):
        tok = 0
        last = -1
        for e in range(counts[b]):
            p, lo, hi, before = blocks[b, e]
            assert 0 <= lo < hi <= P and before == tok
            ts = np.arange(p * P + lo, p * P + hi)
            assert ts[0] > last
            last = ts[-1]
            assert np.all(mem[b, ts] == 0)
            mem[b, ts] = 1
            tok += hi - lo
    return mem


def _oracle_members(lens, Lmax, P, span_lists):
    mem = np.zeros((len(lens), Lmax), dtype=np.uint8)
    for b, L in enumerate(lens):
        mem[b, :L] = oracle.span_members(L, P, span_lists[b])
    return mem


@pytest.mark.parametrize("P", [16, 64])
def test_random_spans_bit_exact(cuda_dev, P):
    rng = np.random.default_rng(P)
    lens = [1, 5, 77, 1000, 4096, 5000]
    Lmax = ((max(lens) + P - 1) // P) * P
    span_lists = []
    for L in lens:
        n = int(rng.integers(0, 9))
        lst = []
        for _ in range(n):
            a = int(rng.integers(-50, L + 50))
            b = a + int(rng.integers(-3, 700))
            lst.append((a, b, bool(rng.integers(0, 2))))
        span_lists.append(lst)
    cache, _ = W.random_decode(1, len(lens), 2, 1, 64, lens, P)
    spans, cnt, rnd = SP.pack(span_lists, cuda_dev)
    ws = sa.Workspace(cuda_dev)
    sel = sa.select_blocks_spans(cache.to(cuda_dev), spans, cnt, rnd, ws=ws)
    ws.raise_on_fault()
    got = _members_from_blocks(sel.blocks.cpu().numpy(), sel.block_counts.cpu().numpy(), P, Lmax)
    want = _oracle_members(lens, Lmax, P, span_lists)
    np.testing.assert_array_equal(got, want)


def test_block_capacity_overflow_is_recorded(cuda_dev):
    cache, _ = W.random_decode(2, 1, 2, 1, 64, [1000], 16)
    spans, cnt, rnd = SP.pack([[(0, 1000, True)]], cuda_dev)
    ws = sa.Workspace(cuda_dev)
    sel = sa.select_blocks_spans(cache.to(cuda_dev), spans, cnt, rnd, max_blocks=10, ws=ws)
    st, det = ws.status()
    assert st == 7 and int(sel.block_counts[0]) == 10


@pytest.mark.parametrize("origin", [0, 5])
def test_masked_decode_modes(cuda_dev, origin):
    """Every mode, ragged lengths, origin offset: block list + decode vs oracle."""
    lens = [3000, 5100, 6000, 2049]
    B, Hq, Hkv, d, P = len(lens), 16, 2, 128, 16
    cache, q = W.random_decode(77 + origin, B, Hq, Hkv, d, lens, P)
    Lmax = cache.max_pages * P
    gc = cache.to(cuda_dev)
    ws = sa.Workspace(cuda_dev)
    scale = 1 / math.sqrt(d)
    for mode, om in [(SP.FOCUS, OM.FOCUS), (SP.LOCAL, OM.LOCAL), (SP.STREAMING, OM.STREAM),
                     (SP.GLOBAL, OM.GLOBAL)]:
        chunks = [(0, 2), (1, 2), (2, 0), (0, 1)]
        prod = [SP.spans_for(mode, L, 2048, origin, chunks[b]) for b, L in enumerate(lens)]
        ref_spans = [OM.mode_spans(om, L, 2048, origin, chunks[b]) for b, L in enumerate(lens)]
        spans, cnt, rnd = SP.pack(prod, cuda_dev)
        sel = sa.select_blocks_spans(gc, spans, cnt, rnd, ws=ws)
        got = _members_from_blocks(sel.blocks.cpu().numpy(), sel.block_counts.cpu().numpy(), P, Lmax)
        want = _oracle_members(lens, Lmax, P, ref_spans)
        np.testing.assert_array_equal(got, want)
        ref, ref_lse = oracle.decode_members(cache, q, want, scale)
        for S in (1, 8):
            out, lse = sa.sparse_decode_attn(gc, q.to(cuda_dev), sel, scale, S, ws=ws)
            assert_close_attn(out.float().cpu().numpy().reshape(-1, d), ref)
            np.testing.assert_allclose(lse.cpu().numpy().reshape(-1), ref_lse, atol=2e-3, rtol=0)
    ws.raise_on_fault()


def test_masked_decode_full_size_steps(cuda_dev):
    """Long-context masked decode at full size (B=4, 64/8 heads, L=131072,
    16-token shuffled pages, 2048-token chunks): a few seeded steps."""
    wl = W.masked_decode(1003, steps=6)
    B, Hq, d, P = 4, 64, 128, 16
    L = 131072
    gc = wl.cache.to(cuda_dev)
    cv = oracle.CacheView(wl.cache)
    ws = sa.Workspace(cuda_dev)
    scale = 1 / math.sqrt(d)
    rows = np.random.default_rng(0).choice(B * Hq, 48, replace=False)
    for step in range(6):
        prod, ref_spans = [], []
        for b in range(B):
            mode = int(wl.modes[step, b])
            ch = wl.focus_chunks[step, b].tolist()
            prod.append(SP.spans_for(SP.MODE_IDS[mode], L, 2048, 0, ch))
            ref_spans.append(OM.mode_spans(mode, L, 2048, 0, ch))
        spans, cnt, rnd = SP.pack(prod, cuda_dev)
        sel = sa.select_blocks_spans(gc, spans, cnt, rnd, ws=ws)
        want = _oracle_members([L] * B, L, P, ref_spans)
        got = _members_from_blocks(sel.blocks.cpu().numpy(), sel.block_counts.cpu().numpy(), P, L)
        np.testing.assert_array_equal(got, want)
        q = wl.q_steps[step]
        out, _ = sa.sparse_decode_attn(gc, q.to(cuda_dev), sel, scale, wl.num_splits, ws=ws)
        ref, _ = oracle.decode_members(cv, q, want, scale, rows=rows)
        assert_close_attn(out.float().cpu().numpy().reshape(-1, d)[rows], ref)
    ws.raise_on_fault()
