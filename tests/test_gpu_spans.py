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
        for S in (1, 8, 64):   # at 64, short lists leave most splits empty
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


@pytest.mark.parametrize("d,Hq,Hkv,qdt", [
    (128, 8, 8, torch.bfloat16),     # one query head per kv head
    (128, 8, 4, torch.bfloat16),
    (128, 16, 4, torch.bfloat16),
    (64, 32, 2, torch.bfloat16),     # 16 query heads per kv head (all MMA rows used)
    (128, 8, 1, torch.float32),      # fp32 query (high + low bf16 parts)
    (128, 32, 1, torch.bfloat16),    # 32 per kv head: per-head kernel
    (128, 12, 1, torch.bfloat16),    # 12 per kv head: two 8-head column blocks, 4 padding heads
    (64, 6, 2, torch.float32),       # 3 per kv head, fp32 query, 5 padding heads
])
def test_masked_decode_group_shapes(cuda_dev, d, Hq, Hkv, qdt):
    lens = [700, 4100, 33, 2500]
    P = 16
    cache, q = W.random_decode(90 + Hq + d, len(lens), Hq, Hkv, d, lens, P, q_dtype=qdt)
    Lmax = cache.max_pages * P
    gc = cache.to(cuda_dev)
    ws = sa.Workspace(cuda_dev)
    scale = 1 / math.sqrt(d)
    prod = [SP.spans_for(SP.GLOBAL, lens[0], 2048), SP.spans_for(SP.FOCUS, lens[1], 2048, 3, [0, 1]),
            SP.spans_for(SP.STREAMING, lens[2], 2048), SP.spans_for(SP.LOCAL, lens[3], 2048)]
    spans, cnt, rnd = SP.pack(prod, cuda_dev)
    sel = sa.select_blocks_spans(gc, spans, cnt, rnd, ws=ws)
    mem = _members_from_blocks(sel.blocks.cpu().numpy(), sel.block_counts.cpu().numpy(), P, Lmax)
    ref, ref_lse = oracle.decode_members(cache, q, mem, scale)
    for S in (1, 3, 8, 37):
        out, lse = sa.sparse_decode_attn(gc, q.to(cuda_dev), sel, scale, S, ws=ws)
        assert_close_attn(out.float().cpu().numpy().reshape(-1, d), ref)
        np.testing.assert_allclose(lse.cpu().numpy().reshape(-1), ref_lse, atol=2e-3, rtol=0)
    ws.raise_on_fault()


@pytest.mark.parametrize("S", [1, 5, 64])
def test_masked_decode_64_token_pages(cuda_dev, S):
    """64-token pages: a split covers at least two list entries, so with many
    splits most of them stay empty and the combine skips them."""
    lens = [3000, 130, 6100]
    P, d, Hq, Hkv = 64, 128, 16, 2
    cache, q = W.random_decode(41 + S, len(lens), Hq, Hkv, d, lens, P)
    Lmax = cache.max_pages * P
    gc = cache.to(cuda_dev)
    ws = sa.Workspace(cuda_dev)
    scale = 1 / math.sqrt(d)
    prod = [SP.spans_for(SP.FOCUS, lens[0], 2048, 7, [0, 1]), SP.spans_for(SP.STREAMING, lens[1], 2048),
            SP.spans_for(SP.LOCAL, lens[2], 2048)]
    spans, cnt, rnd = SP.pack(prod, cuda_dev)
    sel = sa.select_blocks_spans(gc, spans, cnt, rnd, ws=ws)
    mem = _members_from_blocks(sel.blocks.cpu().numpy(), sel.block_counts.cpu().numpy(), P, Lmax)
    ref_spans = [OM.mode_spans(OM.FOCUS, lens[0], 2048, 7, [0, 1]), OM.mode_spans(OM.STREAM, lens[1], 2048),
                 OM.mode_spans(OM.LOCAL, lens[2], 2048)]
    np.testing.assert_array_equal(mem, _oracle_members(lens, Lmax, P, ref_spans))
    ref, ref_lse = oracle.decode_members(cache, q, mem, scale)
    out, lse = sa.sparse_decode_attn(gc, q.to(cuda_dev), sel, scale, S, ws=ws)
    assert_close_attn(out.float().cpu().numpy().reshape(-1, d), ref)
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1), ref_lse, atol=2e-3, rtol=0)
    ws.raise_on_fault()


def test_masked_decode_empty_and_malformed_lists(cuda_dev):
    """An empty list gives a zero output and lse = -inf; a malformed entry is
    recorded as a device fault and skipped, the rest still attends."""
    lens = [500, 900]
    P, d = 16, 128
    cache, q = W.random_decode(5, 2, 8, 1, d, lens, P)
    gc = cache.to(cuda_dev)
    blocks = torch.zeros((2, 4, 4), dtype=torch.int32)
    blocks[1, 0] = torch.tensor([0, 0, 16, 0])
    blocks[1, 1] = torch.tensor([3, 9, 4, 16])       # lo > hi: malformed
    blocks[1, 2] = torch.tensor([5, 2, 10, 16])
    counts = torch.tensor([0, 3], dtype=torch.int32)
    sel = sa.BlockSelection(blocks.to(cuda_dev), counts.to(cuda_dev))
    ws = sa.Workspace(cuda_dev)
    out, lse = sa.sparse_decode_attn(gc, q.to(cuda_dev), sel, 0.1, 2, ws=ws)
    st, det = ws.status()
    assert st == 5 and det[1] == 5            # SA_ERR_DEVICE_FAULT, malformed block entry
    o = out.float().cpu()
    assert torch.all(o[0] == 0) and torch.all(torch.isinf(lse.cpu()[0]))
    mem = np.zeros((2, cache.max_pages * P), dtype=np.uint8)
    mem[1, 0:16] = 1
    mem[1, 5 * 16 + 2:5 * 16 + 10] = 1
    ref, _ = oracle.decode_members(cache, q, mem, 0.1)
    assert_close_attn(o.numpy().reshape(-1, d)[8:], ref.reshape(-1, d)[8:])


def test_da_state_machine_drives_masked_decode(cuda_dev):
    """Scripted tag streams -> host DA state machine -> GPU block lists and
    decode, step by step over growing sequences; the oracle side takes the
    modes written out by hand and builds its spans with oracle.modes."""
    from sparse_attention_aware_b200 import da_state as DA
    V = DA.DAVocab()
    G, LOC, FO, FC = V.global_tag, V.local_tag, V.focus_open, V.focus_close
    C = lambda c: V.chunk_base + c
    prompts = [6000, 9000, 4500]
    streams = [[FO, C(0), C(2), FC, 5, LOC],
               [LOC, 1, G, FO, C(3), FC],
               [7, FO, C(1), FC, G, 2]]
    # mode in effect for each step's read, per the stream above
    modes = [[(OM.GLOBAL, ()), (OM.GLOBAL, ()), (OM.GLOBAL, ()), (OM.FOCUS, (0, 2)), (OM.FOCUS, (0, 2)),
              (OM.LOCAL, ())],
             [(OM.LOCAL, ()), (OM.LOCAL, ()), (OM.GLOBAL, ()), (OM.GLOBAL, ()), (OM.GLOBAL, ()),
              (OM.FOCUS, (3,))],
             [(OM.GLOBAL, ()), (OM.GLOBAL, ()), (OM.GLOBAL, ()), (OM.FOCUS, (1,)), (OM.GLOBAL, ()),
              (OM.GLOBAL, ())]]
    steps = 6
    Hq, Hkv, d, P = 16, 2, 128, 16
    cap = [L + steps for L in prompts]
    cache, _ = W.random_decode(123, len(prompts), Hq, Hkv, d, cap, P)
    Lmax = cache.max_pages * P
    g = torch.Generator().manual_seed(321)
    machine = DA.DABatch(prompts)
    ws = sa.Workspace(cuda_dev)
    scale = 1 / math.sqrt(d)
    for i in range(steps):
        lens = [L + i + 1 for L in prompts]
        step_cache = W.PagedCache(cache.k, cache.v, cache.page_table, torch.tensor(lens, dtype=torch.int32))
        gc = step_cache.to(cuda_dev)
        spans, cnt, rnd = machine.step([s[i] for s in streams], lens, device=cuda_dev)
        sel = sa.select_blocks_spans(gc, spans, cnt, rnd, ws=ws)
        want = np.zeros((len(prompts), Lmax), dtype=np.uint8)
        for b, L in enumerate(lens):
            m, ch = modes[b][i]
            want[b, :L] = oracle.span_members(L, P, OM.mode_spans(m, L, 2048, 0, ch))
        got = _members_from_blocks(sel.blocks.cpu().numpy(), sel.block_counts.cpu().numpy(), P, Lmax)
        np.testing.assert_array_equal(got, want)
        q = torch.randn((len(prompts), Hq, d), generator=g).to(torch.bfloat16)
        out, lse = sa.sparse_decode_attn(gc, q.to(cuda_dev), sel, scale, 4, ws=ws)
        ref, ref_lse = oracle.decode_members(step_cache, q, want, scale)
        assert_close_attn(out.float().cpu().numpy().reshape(-1, d), ref)
        np.testing.assert_allclose(lse.cpu().numpy().reshape(-1), ref_lse, atol=2e-3, rtol=0)
    ws.raise_on_fault()


def test_span_packer_matches_pack_over_steps(cuda_dev):
    """The non-blocking packer gives the same device tensors as pack() for a
    run of steps, with its pinned buffers reused (depth 2) and the previous
    step's selection still queued when the next step is packed."""
    rng = np.random.default_rng(5)
    cache, _ = W.random_decode(9, 3, 2, 1, 64, [3000, 4096, 777], 16)
    gc = cache.to(cuda_dev)
    packer = SP.SpanPacker(3, 2, cuda_dev)
    ws = sa.Workspace(cuda_dev)
    for step in range(6):
        lists = []
        for L in (3000, 4096, 777):
            n = int(rng.integers(0, 3))
            lists.append([(int(a), int(a) + int(rng.integers(1, 900)), bool(rng.integers(0, 2)))
                          for a in rng.integers(-20, L, n)])
        want = SP.pack(lists, cuda_dev, max_spans=2)
        got = packer.pack(lists)
        sel_w = sa.select_blocks_spans(gc, *want, ws=ws)
        sel_g = sa.select_blocks_spans(gc, *got, ws=ws)
        torch.cuda.synchronize()
        for x, y in zip(got, want):
            assert torch.equal(x, y)
        assert torch.equal(sel_g.block_counts, sel_w.block_counts)
        for b, n in enumerate(sel_w.block_counts.tolist()):    # entries past a count are not written
            assert torch.equal(sel_g.blocks[b, :n], sel_w.blocks[b, :n])
