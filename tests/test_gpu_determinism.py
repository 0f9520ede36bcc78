"""Run-to-run bitwise determinism of every op (fixed split, reduction and
selection orders; integer-only atomics): each call is made twice on the same
inputs and the outputs must be identical bit for bit."""
import math

import pytest
import torch

import sparse_attention_aware_b200 as sa
from sparse_attention_aware_b200 import spans as SP
from sparse_attention_aware_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _twice(fn):
    a = fn()
    torch.cuda.synchronize()
    a = [x.clone() for x in a]
    b = fn()
    torch.cuda.synchronize()
    return a, b


def test_topk_and_token_decode_deterministic(cuda_dev):
    cache, q = W.random_decode(21, 4, 16, 4, 128, [5000, 3000, 7000, 6500], 16)
    gc, gq = cache.to(cuda_dev), q.to(cuda_dev)
    ws = sa.Workspace(cuda_dev)

    def run():
        sel = sa.select_topk(gc, gq, 300, ws=ws)
        out, lse = sa.sparse_decode_attn(gc, gq, sel, 0.1, 8, ws=ws)
        return [sel.idx, sel.count, out, lse]

    a, b = _twice(run)
    assert all(torch.equal(x, y) for x, y in zip(a, b))


def test_span_blocks_and_group_decode_deterministic(cuda_dev):
    lens = [9000, 12000, 700]
    cache, q = W.random_decode(22, 3, 32, 4, 128, lens, 16)
    gc, gq = cache.to(cuda_dev), q.to(cuda_dev)
    prod = [SP.spans_for(SP.FOCUS, lens[0], 2048, 0, [1, 3]), SP.spans_for(SP.GLOBAL, lens[1]),
            SP.spans_for(SP.STREAMING, lens[2])]
    spans, cnt, rnd = SP.pack(prod, cuda_dev)
    ws = sa.Workspace(cuda_dev)

    def run():
        sel = sa.select_blocks_spans(gc, spans, cnt, rnd, ws=ws)
        out, lse = sa.sparse_decode_attn(gc, gq, sel, 0.1, 8, ws=ws)
        return [sel.block_counts, out, lse]

    a, b = _twice(run)
    assert all(torch.equal(x, y) for x, y in zip(a, b))


def test_rbs_and_prefill_deterministic(cuda_dev):
    wl = W.clustered_prefill(23, T=4096 + 100, Hq=8, Hkv=2, d=128, block=64, n_clusters=16)
    gc, gq = wl.cache.to(cuda_dev), wl.q.to(cuda_dev)
    ws = sa.Workspace(cuda_dev)
    scale = 1 / math.sqrt(128)

    def run():
        csr = sa.select_blocks_rbs(gc, gq, 64, scale, p_c=0.9, p_r=0.93, ws=ws)
        out, lse = sa.sparse_prefill_attn(gc, gq, csr, scale, ws=ws)
        n = int(csr.row_ptr[-1])
        return [csr.row_ptr, csr.cols[:n], csr.tau, out, lse]

    a, b = _twice(run)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
