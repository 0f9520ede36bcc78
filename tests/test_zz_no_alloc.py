"""The allocation-free decode entry point, called through the C ABI.

sa_sparse_decode_attn_noalloc is for callers that cannot allocate device
memory (a plugin handed only its input and output buffers by its host engine,
or a serving loop that must not call an allocator), so they cannot pass the
workspace the regular decode entry point needs.  Its scratch is a fixed
8 MiB device array inside the library.

The header promises the same results as sa_sparse_decode_attn, bit for bit,
so outputs and LSE are compared with torch.equal, on two calls in a row
(different problems, so a stale scratch from the first call would show in
the second), for token-list selections (per-head split kernel) and for
block-list selections (the GQA group kernel), where the second call's lists
are short enough that it leaves some of the first call's splits untouched.
One case of each is also checked against the CPU oracle within the stated
tolerance.  The file is named so that pytest collects it last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_aware_b200 as sa
from oracle import modes as OM
from sparse_attention_aware_b200 import _lib as L
from sparse_attention_aware_b200 import spans as SP
from sparse_attention_aware_b200 import workloads as W
from sparse_attention_aware_b200.api import kv_struct
from tests.helpers import assert_close_attn

pytestmark = pytest.mark.gpu


def _problem(seed, B, Hq, Hkv, lens, kcap, counts):
    cache, q = W.random_decode(seed, B, Hq, Hkv, 128, lens, 16)
    rng = np.random.default_rng(seed)
    idx = np.full((B, Hq, kcap), -1, dtype=np.int32)
    cnt = np.zeros((B, Hq), dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            n = min(counts[(b * Hq + h) % len(counts)], lens[b])
            idx[b, h, :n] = np.sort(rng.choice(lens[b], n, replace=False))
            cnt[b, h] = n
    return cache, q, idx, cnt


def _noalloc(lib, cache, q, sel, scale, splits, out, lse):
    kv = kv_struct(cache, q.device)
    s = sel.struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.sa_sparse_decode_attn_noalloc(ctypes.byref(kv), ctypes.c_void_p(q.data_ptr()), L.DTYPE_BF16,
                                             q.shape[1], ctypes.byref(s), scale, splits,
                                             ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
                                             stream)


def _both(lib, gc, qd, sel, scale, splits):
    """(workspace entry point, allocation-free entry point) results."""
    ref, ref_lse = sa.sparse_decode_attn(gc, qd, sel, scale, splits, ws=sa.Workspace(qd.device))
    out = torch.full_like(ref, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    assert _noalloc(lib, gc, qd, sel, scale, splits, out, lse) == 0
    torch.cuda.synchronize()
    return ref, ref_lse, out, lse


def test_noalloc_token_lists_bitwise_twice(cuda_dev):
    lib = L.load()
    cases = [(71, 8, 32, 8, [4000, 333, 2500, 1, 4096, 3000, 17, 1500], 1024, [1024, 0, 7, 900], 8),
             (72, 3, 16, 4, [900, 5000, 64], 700, [700, 3, 650], 3)]
    for n, (seed, B, Hq, Hkv, lens, kcap, counts, splits) in enumerate(cases):
        cache, q, idx, cnt = _problem(seed, B, Hq, Hkv, lens, kcap, counts)
        gc, qd = cache.to(cuda_dev), q.to(cuda_dev)
        sel = sa.TokenSelection(torch.from_numpy(idx).to(cuda_dev), torch.from_numpy(cnt).to(cuda_dev))
        scale = 1 / math.sqrt(128)
        ref, ref_lse, out, lse = _both(lib, gc, qd, sel, scale, splits)
        assert torch.equal(out, ref)
        assert torch.equal(lse, ref_lse)
        if n == 1:
            want, want_lse = oracle.decode_tokens(cache, q, idx, cnt, scale)
            assert_close_attn(out.float().cpu().numpy().reshape(-1, 128), want)
            got_lse = lse.cpu().numpy().reshape(-1).astype(np.float64)
            fin = np.isfinite(want_lse)
            assert np.array_equal(np.isfinite(got_lse), fin)
            assert np.abs(got_lse[fin] - want_lse[fin]).max() <= 2e-3


def test_noalloc_block_lists_bitwise_twice(cuda_dev):
    """GQA block-list kernel: the first call's long lists use every split, the
    second call's short lists (DA local / LoZA streaming windows) leave most
    splits empty, so the scratch still holds the first call's partial states
    where the second call writes none."""
    lib = L.load()
    scale = 1 / math.sqrt(128)
    lens = [6000, 8192, 3001]
    cache, q = W.random_decode(81, 3, 32, 4, 128, lens, 16)
    gc, qd = cache.to(cuda_dev), q.to(cuda_dev)
    calls = [[SP.spans_for(SP.GLOBAL, L_) for L_ in lens],
             [SP.spans_for(SP.LOCAL, lens[0]), SP.spans_for(SP.STREAMING, lens[1]), SP.spans_for(SP.LOCAL, lens[2])]]
    om = [[OM.mode_spans(OM.GLOBAL, L_) for L_ in lens],
          [OM.mode_spans(OM.LOCAL, lens[0]), OM.mode_spans(OM.STREAM, lens[1]), OM.mode_spans(OM.LOCAL, lens[2])]]
    for n, lists in enumerate(calls):
        spans, cnt, rnd = SP.pack(lists, cuda_dev)
        ws = sa.Workspace(cuda_dev)
        bsel = sa.select_blocks_spans(gc, spans, cnt, rnd, ws=ws)
        ws.raise_on_fault("spans")
        ref, ref_lse, out, lse = _both(lib, gc, qd, bsel, scale, 16)
        assert torch.equal(out, ref)
        assert torch.equal(lse, ref_lse)
        if n == 1:
            Lmax = cache.max_pages * 16
            member = np.zeros((3, Lmax), dtype=np.uint8)
            for b, L_ in enumerate(lens):
                member[b, :L_] = oracle.span_members(L_, 16, om[n][b])
            want, want_lse = oracle.decode_members(cache, q, member, scale)
            assert_close_attn(out.float().cpu().numpy().reshape(-1, 128), want)
            got_lse = lse.cpu().numpy().reshape(-1).astype(np.float64)
            assert np.abs(got_lse - want_lse).max() <= 2e-3


def test_noalloc_decode_rejects_problems_beyond_its_scratch(cuda_dev):
    lib = L.load()
    # 64 sequences x 64 heads x 8 splits x (128 + 2) x 4 B is about 17 MB > 8 MiB
    cache, q = W.random_decode(5, 64, 64, 8, 128, [16] * 64, 16)
    gc = cache.to(cuda_dev)
    qd = q.to(cuda_dev)
    idx = torch.zeros((64, 64, 1), dtype=torch.int32, device=cuda_dev)
    cnt = torch.ones((64, 64), dtype=torch.int32, device=cuda_dev)
    out = torch.empty((64, 64, 128), dtype=torch.bfloat16, device=cuda_dev)
    lse = torch.empty((64, 64), dtype=torch.float32, device=cuda_dev)
    assert _noalloc(lib, gc, qd, sa.TokenSelection(idx, cnt), 0.1, 8, out, lse) == 2   # SA_ERR_UNSUPPORTED
