"""ctypes declarations of libsa's C ABI (include/sa.h).  Marshalling only."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsa.so")

c_i32 = ctypes.c_int32
c_f32 = ctypes.c_float
c_vp = ctypes.c_void_p
c_size = ctypes.c_size_t

SA_OK = 0
STATUS_NAMES = {0: "SA_OK", 1: "SA_ERR_INVALID_ARGUMENT", 2: "SA_ERR_UNSUPPORTED",
                3: "SA_ERR_WORKSPACE", 4: "SA_ERR_CUDA", 5: "SA_ERR_DEVICE_FAULT",
                6: "SA_ERR_TIMEOUT", 7: "SA_ERR_CAPACITY"}
DTYPE_F32, DTYPE_BF16 = 0, 1
SEL_TOKENS, SEL_BLOCKS = 1, 2
SEL_RBS, SEL_SPANS = 1, 2
OP_SELECT_TOPK, OP_SELECT_BLOCKS, OP_DECODE, OP_PREFILL = 1, 2, 3, 4

EXPORTS = ("sa_select_topk", "sa_select_blocks", "sa_sparse_decode_attn", "sa_sparse_prefill_attn",
           "sa_workspace_bytes", "sa_workspace_init", "sa_read_device_status", "sa_status_string",
           "sa_version", "sa_sparse_decode_attn_noalloc", "sa_fetch_pages", "sa_tier_plan",
           "sa_tier_plan_scratch_ints", "sa_check_bounded_wait")


class KVCacheS(ctypes.Structure):
    _fields_ = [("k", c_vp), ("v", c_vp), ("page_table", c_vp), ("seq_lens", c_vp),
                ("batch", c_i32), ("num_kv_heads", c_i32), ("head_dim", c_i32),
                ("page_size", c_i32), ("max_pages_per_seq", c_i32), ("num_pages", c_i32)]


class SelectionS(ctypes.Structure):
    _fields_ = [("kind", c_i32), ("idx", c_vp), ("count", c_vp), ("k_cap", c_i32),
                ("blocks", c_vp), ("block_counts", c_vp), ("max_blocks", c_i32)]


class BlockSelectArgsS(ctypes.Structure):
    _fields_ = [("mode", c_i32), ("q", c_vp), ("num_q_heads", c_i32), ("num_tokens", c_i32),
                ("block_size", c_i32), ("scale", c_f32), ("tau_c", c_vp), ("tau_r", c_vp),
                ("p_c", c_f32), ("p_r", c_f32), ("force_diag", c_i32), ("force_first", c_i32),
                ("spans", c_vp), ("span_counts", c_vp), ("span_round", c_vp), ("max_spans", c_i32)]


class BlockListS(ctypes.Structure):
    _fields_ = [("row_ptr", c_vp), ("cols", c_vp), ("nnz_capacity", ctypes.c_int64),
                ("tau_out", c_vp), ("blocks", c_vp), ("block_counts", c_vp), ("max_blocks", c_i32)]


class WsQueryS(ctypes.Structure):
    _fields_ = [("num_q_heads", c_i32), ("k", c_i32), ("num_splits", c_i32), ("num_tokens", c_i32),
                ("block_args", ctypes.POINTER(BlockSelectArgsS))]


_lib = None


def load(path: str = LIB_PATH):
    """Load libsa.so.  Raises if the CUDA library has not been built: there is
    no fallback implementation."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            "libsa.so not found at %s: build it with `python -m sparse_attention_aware_b200.build` "
            "(the CUDA library is required; there is no CPU fallback)" % path)
    L = ctypes.CDLL(path)
    P = ctypes.POINTER
    L.sa_select_topk.argtypes = [P(KVCacheS), c_vp, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_size, c_vp]
    L.sa_select_blocks.argtypes = [P(KVCacheS), P(BlockSelectArgsS), P(BlockListS), c_vp, c_size, c_vp]
    L.sa_sparse_decode_attn.argtypes = [P(KVCacheS), c_vp, c_i32, c_i32, P(SelectionS), c_f32, c_i32,
                                        c_vp, c_vp, c_vp, c_size, c_vp]
    L.sa_sparse_decode_attn_noalloc.argtypes = [P(KVCacheS), c_vp, c_i32, c_i32, P(SelectionS), c_f32, c_i32,
                                                c_vp, c_vp, c_vp]
    L.sa_fetch_pages.argtypes = [c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, ctypes.c_int64, ctypes.c_int64, c_size,
                                 c_vp, c_size, c_vp]
    L.sa_sparse_prefill_attn.argtypes = [P(KVCacheS), c_vp, c_i32, c_i32, P(BlockListS), c_f32, c_i32,
                                         c_vp, c_vp, c_vp, c_size, c_vp]
    L.sa_tier_plan.argtypes = [c_vp, ctypes.c_int64, c_vp, c_vp, c_i32, ctypes.c_int64, c_vp, c_i32, c_vp, c_i32,
                               c_vp, c_vp, c_vp, c_vp, ctypes.c_int64]
    L.sa_check_bounded_wait.argtypes = [ctypes.c_int64, c_vp, c_size, c_vp]
    L.sa_tier_plan_scratch_ints.argtypes = [ctypes.c_int64, c_i32]
    L.sa_tier_plan_scratch_ints.restype = ctypes.c_int64
    L.sa_workspace_bytes.argtypes = [c_i32, P(KVCacheS), P(WsQueryS)]
    L.sa_workspace_bytes.restype = c_size
    L.sa_workspace_init.argtypes = [c_vp, c_size, c_vp]
    L.sa_read_device_status.argtypes = [c_vp, c_vp, P(c_i32)]
    L.sa_status_string.argtypes = [c_i32]
    L.sa_status_string.restype = ctypes.c_char_p
    L.sa_version.restype = c_i32
    for fn in ("sa_select_topk", "sa_select_blocks", "sa_sparse_decode_attn", "sa_sparse_prefill_attn",
               "sa_workspace_init", "sa_read_device_status", "sa_sparse_decode_attn_noalloc", "sa_fetch_pages",
               "sa_tier_plan", "sa_check_bounded_wait"):
        getattr(L, fn).restype = c_i32
    _lib = L
    return L
