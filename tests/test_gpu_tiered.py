"""GPU: host-tier page fetch and tiered-KV masked decode.

The tiered cache must give bit-identical results to the fully resident cache:
same kernels, same bytes, only the page slots differ."""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_aware_b200 as sa
from sparse_attention_aware_b200 import da_state as DA
from sparse_attention_aware_b200 import spans as SP
from sparse_attention_aware_b200 import tiered as T
from sparse_attention_aware_b200 import workloads as W
from tests.helpers import assert_close_attn

pytestmark = pytest.mark.gpu


def test_fetch_pages_copies_whole_pages_and_records_bad_pairs(cuda_dev):
    g = torch.Generator().manual_seed(5)
    host_k = torch.randn((40, 2, 16, 128), generator=g).to(torch.bfloat16).pin_memory()
    host_v = torch.randn((40, 2, 16, 128), generator=g).to(torch.bfloat16).pin_memory()
    dev_k = torch.zeros((12, 2, 16, 128), dtype=torch.bfloat16, device=cuda_dev)
    dev_v = torch.zeros_like(dev_k)
    src = [3, 39, 0, 17, 22]
    dst = [11, 0, 5, 2, 7]
    pairs = torch.tensor(list(zip(src, dst)), dtype=torch.int32, device=cuda_dev)
    ws = sa.Workspace(cuda_dev)
    sa.fetch_pages(host_k, host_v, dev_k, dev_v, pairs, ws=ws)
    ws.raise_on_fault()
    for s_, d_ in zip(src, dst):
        assert torch.equal(dev_k[d_].cpu(), host_k[s_]) and torch.equal(dev_v[d_].cpu(), host_v[s_])
    untouched = [i for i in range(12) if i not in dst]
    assert torch.all(dev_k[untouched] == 0)
    bad = torch.tensor([[40, 1], [4, 12], [6, 4]], dtype=torch.int32, device=cuda_dev)
    sa.fetch_pages(host_k, host_v, dev_k, dev_v, bad, ws=ws)
    st, det = ws.status()
    assert st == 5 and det[1] == 2                       # SA_ERR_DEVICE_FAULT, page check
    assert torch.equal(dev_k[4].cpu(), host_k[6])         # the good pair still lands
    with pytest.raises(ValueError):
        sa.fetch_pages(host_k.clone(), host_v, dev_k, dev_v, pairs)   # not pinned


def test_tiered_masked_decode_is_bitwise_the_resident_decode(cuda_dev):
    """A DA tag stream over 3 sequences with a device pool of half of the
    pages and lengths published by the tier each step: every step's block
    list and decode equal those of the fully resident cache bit for bit, and
    the oracle agrees."""
    V = DA.DAVocab()
    G, LOC, FO, FC = V.global_tag, V.local_tag, V.focus_open, V.focus_close
    C = lambda c: V.chunk_base + c
    P, Hq, Hkv, d = 16, 16, 2, 128
    # sequence 0's first focus chunk (5) runs past its decode length: the
    # pages past the length are neither requested nor read
    prompts = [11990, 9000, 10000]
    streams = [[LOC, FO, C(5), FC, FO, C(1), C(4), FC, 3, FO, C(0), FC, LOC, 5],
               [FO, C(2), FC, 1, LOC, 2, FO, C(3), C(1), FC, 4, 5, LOC, 6],
               [LOC, 1, 2, FO, C(0), C(3), FC, 3, 4, LOC, FO, C(4), FC, 7]]
    steps = len(streams[0])
    cap = [L + steps for L in prompts]
    full, _ = W.random_decode(77, 3, Hq, Hkv, d, cap, P)
    pages_total = sum((L + P - 1) // P for L in cap)
    tier = T.TieredKV(full, slots=int(0.5 * pages_total), device=cuda_dev)
    res = full.to(cuda_dev)
    machine = DA.DABatch(prompts)
    ws_t, ws_r = sa.Workspace(cuda_dev), sa.Workspace(cuda_dev)
    g = torch.Generator().manual_seed(9)
    scale = 1 / math.sqrt(d)
    fetched = 0
    for i in range(steps):
        lens = [L + i + 1 for L in prompts]
        lens_t = torch.tensor(lens, dtype=torch.int32, device=cuda_dev)
        lists = []
        for b, m in enumerate(machine.machines):
            m.observe(streams[b][i])
            lists.append(m.next_spans(lens[b]))
        spans, cnt, rnd = SP.pack(lists, cuda_dev, max_spans=2)
        if i % 2:   # both entry points: page lists, and span lists mapped range by range
            fetched += tier.prepare_spans(lists, lens)
        else:
            fetched += tier.prepare([T.span_pages(l, L, P) for l, L in zip(lists, lens)], seq_lens=lens)
        tc = tier.cache
        assert torch.equal(tc.seq_lens, lens_t)
        rc = W.PagedCache(res.k, res.v, res.page_table, lens_t)
        sel_t = sa.select_blocks_spans(tc, spans, cnt, rnd, ws=ws_t)
        sel_r = sa.select_blocks_spans(rc, spans, cnt, rnd, ws=ws_r)
        assert torch.equal(sel_t.block_counts, sel_r.block_counts)
        for b, n in enumerate(sel_t.block_counts.tolist()):
            assert torch.equal(sel_t.blocks[b, :n], sel_r.blocks[b, :n])
        q = torch.randn((3, Hq, d), generator=g).to(torch.bfloat16).to(cuda_dev)
        o_t, l_t = sa.sparse_decode_attn(tc, q, sel_t, scale, 4, ws=ws_t)
        o_r, l_r = sa.sparse_decode_attn(rc, q, sel_r, scale, 4, ws=ws_r)
        assert torch.equal(o_t, o_r) and torch.equal(l_t, l_r)
        if i == steps - 1:
            mem = np.zeros((3, full.max_pages * P), dtype=np.uint8)
            for b, L in enumerate(lens):
                mem[b, :L] = oracle.span_members(L, P, lists[b])
            cpu_cache = W.PagedCache(full.k, full.v, full.page_table, torch.tensor(lens, dtype=torch.int32))
            ref, _ = oracle.decode_members(cpu_cache, q.cpu(), mem, scale)
            assert_close_attn(o_t.float().cpu().numpy().reshape(-1, d), ref)
    ws_t.raise_on_fault()
    ws_r.raise_on_fault()
    st = tier.map.stats
    assert st["misses"] == fetched > 0 and st["hits"] > 0
    assert len(tier.map.page_in) == tier.map.slots < pages_total


def test_tiered_pool_too_small_for_a_global_step(cuda_dev):
    full, _ = W.random_decode(3, 1, 4, 1, 128, [5000], 16)
    tier = T.TieredKV(full, slots=100, device=cuda_dev)
    with pytest.raises(RuntimeError):
        tier.prepare([T.span_pages(SP.spans_for(SP.GLOBAL, 5000), 5000, 16)])
