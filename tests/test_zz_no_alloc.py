"""The allocation-free decode entry point, called through the C ABI.

sa_sparse_decode_attn_noalloc is for callers that cannot allocate device
memory (a plugin handed only its input and output buffers by its host engine,
or a serving loop that must not call an allocator), so they cannot pass the
workspace the regular decode entry point needs.  Its scratch is a fixed
8 MiB device array inside the library.  This test compares it with the
regular entry point on two calls in a row (different problems, so a stale
scratch from the first call would show in the second) and checks the size
limit.  The file is named so that pytest collects it last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import sparse_attention_aware_b200 as sa
from sparse_attention_aware_b200 import _lib as L
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
    kv = kv_struct(cache)
    s = sel.struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.sa_sparse_decode_attn_noalloc(ctypes.byref(kv), ctypes.c_void_p(q.data_ptr()), L.DTYPE_BF16,
                                             q.shape[1], ctypes.byref(s), scale, splits,
                                             ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
                                             stream)


def test_noalloc_decode_matches_workspace_decode_twice(cuda_dev):
    lib = L.load()
    cases = [(71, 8, 32, 8, [4000, 333, 2500, 1, 4096, 3000, 17, 1500], 1024, [1024, 0, 7, 900], 8),
             (72, 3, 16, 4, [900, 5000, 64], 700, [700, 3, 650], 3)]
    for seed, B, Hq, Hkv, lens, kcap, counts, splits in cases:
        cache, q, idx, cnt = _problem(seed, B, Hq, Hkv, lens, kcap, counts)
        gc = cache.to(cuda_dev)
        qd = q.to(cuda_dev)
        sel = sa.TokenSelection(torch.from_numpy(idx).to(cuda_dev), torch.from_numpy(cnt).to(cuda_dev))
        scale = 1 / math.sqrt(128)
        ref, ref_lse = sa.sparse_decode_attn(gc, qd, sel, scale, splits, ws=sa.Workspace(cuda_dev))
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert _noalloc(lib, gc, qd, sel, scale, splits, out, lse) == 0
        torch.cuda.synchronize()
        assert_close_attn(out.float().cpu().numpy().reshape(-1, 128), ref.float().cpu().numpy().reshape(-1, 128))
        fin = torch.isfinite(ref_lse)
        assert torch.equal(torch.isfinite(lse), fin)
        assert (lse[fin] - ref_lse[fin]).abs().max().item() <= 2e-3


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
