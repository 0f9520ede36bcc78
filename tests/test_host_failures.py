"""Host-side failure injection through the binding (CPU): a workspace that
cannot be allocated, a too-small workspace, and a misaligned workspace fail
with a clear error before anything is launched."""
import ctypes

import pytest
import torch

import sparse_attention_aware_b200 as sa
from sparse_attention_aware_b200 import _lib as L
from sparse_attention_aware_b200 import api
from sparse_attention_aware_b200 import workloads as W


def _cache():
    return W.random_decode(3, 1, 4, 1, 64, [100], 16)


def test_workspace_allocation_failure_propagates(monkeypatch):
    cache, q = _cache()

    def fail(self, nbytes):
        raise MemoryError("injected: device workspace allocation failed")

    monkeypatch.setattr(api.Workspace, "get", fail)
    with pytest.raises(MemoryError, match="injected"):
        sa.select_topk(cache, q, 8, ws=api.Workspace("cpu"))
    with pytest.raises(MemoryError, match="injected"):
        idx = torch.zeros((1, 4, 8), dtype=torch.int32)
        sa.sparse_decode_attn(cache, q, sa.TokenSelection(idx, torch.zeros((1, 4), dtype=torch.int32)),
                              0.1, 2, ws=api.Workspace("cpu"))


def test_small_or_misaligned_workspace_is_rejected_before_launch():
    lib = L.load()
    cache, q = _cache()
    kv = api.kv_struct(cache)
    need = api.workspace_bytes(L.OP_SELECT_TOPK, cache, num_q_heads=4, k=8)
    WS = 3
    buf = ctypes.create_string_buffer(need + 512)
    base = (ctypes.addressof(buf) + 255) // 256 * 256
    idx = ctypes.create_string_buffer(4 * 4 * 8 + 64)
    cnt = ctypes.create_string_buffer(4 * 4 + 64)
    ia = (ctypes.addressof(idx) + 15) // 16 * 16
    ca = (ctypes.addressof(cnt) + 15) // 16 * 16
    qa = q.contiguous()
    # too small by one byte, and misaligned: host checks fail, nothing is launched
    assert lib.sa_select_topk(ctypes.byref(kv), qa.data_ptr(), L.DTYPE_F32, 4, 8, ia, ca, base, need - 1, None) == WS
    assert lib.sa_select_topk(ctypes.byref(kv), qa.data_ptr(), L.DTYPE_F32, 4, 8, ia, ca, base + 8, need, None) == WS
