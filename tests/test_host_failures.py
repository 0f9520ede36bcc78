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

    def fail(self, nbytes, stream=None):
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


def test_caller_tensors_with_the_wrong_layout_are_rejected_before_launch():
    """Outputs the caller provides must have the exact layout the library
    writes; the RBS selection and the prefill take bf16 queries only."""
    cache, q = _cache()                       # B=1, Hq=4, d=64
    with pytest.raises(ValueError, match="select_topk idx"):
        sa.select_topk(cache, q, 8, idx=torch.zeros((1, 4, 9), dtype=torch.int32))
    with pytest.raises(ValueError, match="select_topk count"):
        sa.select_topk(cache, q, 8, count=torch.zeros((1, 4), dtype=torch.int64))
    idx = torch.zeros((1, 4, 8), dtype=torch.int32)
    sel = sa.TokenSelection(idx, torch.zeros((1, 4), dtype=torch.int32))
    with pytest.raises(ValueError, match="sparse_decode_attn out"):
        sa.sparse_decode_attn(cache, q, sel, 0.1, 2, out=torch.zeros((1, 4, 64), dtype=torch.float32))
    with pytest.raises(ValueError, match="sparse_decode_attn lse"):
        sa.sparse_decode_attn(cache, q, sel, 0.1, 2, lse=torch.zeros((4, 1), dtype=torch.float32))
    wl = W.random_prefill(5, 200, 2, 1, 128, 64)
    with pytest.raises(TypeError, match="bf16"):
        sa.select_blocks_rbs(wl.cache, wl.q.float(), 64, tau_c=0.0, tau_r=0.0)
    csr = sa.BlockCSR(torch.zeros(2 * 4 + 1, dtype=torch.int32), torch.zeros(8, dtype=torch.int32),
                      torch.zeros((2, 2)), 2, 4)
    with pytest.raises(TypeError, match="bf16"):
        sa.sparse_prefill_attn(wl.cache, wl.q.float(), csr)
    with pytest.raises(ValueError, match="csr.row_ptr"):
        sa.sparse_prefill_attn(wl.cache, wl.q, sa.BlockCSR(torch.zeros(5, dtype=torch.int32), csr.cols, csr.tau, 2, 4))
    with pytest.raises(ValueError, match="sparse_prefill_attn out"):
        sa.sparse_prefill_attn(wl.cache, wl.q, csr, out=torch.zeros((200, 2, 128), dtype=torch.bfloat16)[:, :1])


def test_selection_tensors_with_the_wrong_layout_are_rejected_before_launch():
    """The decode reads the selection tensors by the (B, Hq) shape of its
    queries: a short count, a wide index type, a non-contiguous index or a
    block list of the wrong width must raise before anything is launched."""
    cache, q = _cache()                       # B=1, Hq=4
    idx = torch.zeros((1, 4, 8), dtype=torch.int32)
    cnt = torch.zeros((1, 4), dtype=torch.int32)
    bad = [
        (sa.TokenSelection(idx, torch.zeros((1, 3), dtype=torch.int32)), "TokenSelection.count"),
        (sa.TokenSelection(idx.long(), cnt), "TokenSelection.idx"),
        (sa.TokenSelection(torch.zeros((1, 8, 4), dtype=torch.int32).transpose(1, 2), cnt), "TokenSelection.idx"),
        (sa.TokenSelection(torch.zeros((2, 4, 8), dtype=torch.int32), cnt), "TokenSelection.idx"),
        (sa.BlockSelection(torch.zeros((1, 5, 3), dtype=torch.int32), torch.zeros((1,), dtype=torch.int32)),
         "BlockSelection.blocks"),
        (sa.BlockSelection(torch.zeros((1, 5, 4), dtype=torch.int32), torch.zeros((2,), dtype=torch.int32)),
         "BlockSelection.block_counts"),
    ]
    for sel, what in bad:
        with pytest.raises(ValueError, match=what):
            sa.sparse_decode_attn(cache, q, sel, 0.1, 2)
    with pytest.raises(TypeError, match="TokenSelection or a BlockSelection"):
        sa.sparse_decode_attn(cache, q, (idx, cnt), 0.1, 2)


def test_cache_descriptors_are_checked_without_asserts():
    """kv_struct raises ValueError (not assert, which python -O drops) for a
    short seq_lens, a wrong dtype, or cache tensors on another device."""
    import dataclasses
    cache, q = _cache()
    short = dataclasses.replace(cache, seq_lens=torch.zeros((0,), dtype=torch.int32))
    with pytest.raises(ValueError, match="seq_lens"):
        api.kv_struct(short)
    with pytest.raises(ValueError, match="bf16"):
        api.kv_struct(dataclasses.replace(cache, k=cache.k.float()))
    with pytest.raises(ValueError, match="page_table"):
        api.kv_struct(dataclasses.replace(cache, page_table=cache.page_table.long()))
    with pytest.raises(ValueError, match="one device"):
        api.kv_struct(cache, torch.device("meta"))
