"""Head-aware sparse attention over a paged bf16 KV cache, B200-native.

The compute lives in ``libsa.so`` (hand-written sm_100a CUDA behind a C ABI,
``include/sa.h``); this package is its ctypes binding plus the seeded
workload generators.  Build the library with
``python -m sparse_attention_aware_b200.build``.
"""
from .api import (BlockCSR, BlockSelection, SAError, TokenSelection, Workspace, check_bounded_wait, fetch_pages,
                  select_blocks_rbs,
                  select_blocks_spans, select_topk, sparse_decode_attn, sparse_prefill_attn,
                  workspace_bytes)
from .cache import PagedCache

__all__ = ["select_topk", "select_blocks_rbs", "select_blocks_spans", "sparse_decode_attn",
           "sparse_prefill_attn", "workspace_bytes", "Workspace", "TokenSelection", "BlockSelection",
           "BlockCSR", "SAError", "fetch_pages", "check_bounded_wait", "PagedCache"]
