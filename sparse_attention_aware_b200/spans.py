"""Host-side construction of span lists for the block-aligned decode modes.

A mode is turned into token ranges that ``select_blocks_spans`` rounds,
clips, merges and lays out per page on the GPU:

* DA ``<global>`` -- all of the context ("百万上下文，模型终于会挑重点了",
  section "三种模式，背后是三种推理状态");
* DA ``<focus>`` -- the declared chunks; chunks are the ~2048-token "magic
  chunks" ("语言模型能自己决定该看哪里吗？", section on the DA protocol), kept
  ranges rounded out to page edges (DA state machine section);
* DA ``<local>`` -- recent tokens only, read as the last 512 tokens, rounded
  out like focus;
* LoZA streaming -- a fixed window over the last 1024 tokens
  ("稀疏注意力机制创新…", section "二、ZigZag架构") plus 4 sink tokens,
  token-exact.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch

GLOBAL, FOCUS, LOCAL, STREAMING = "global", "focus", "local", "streaming"
MODE_IDS = {0: FOCUS, 1: LOCAL, 2: STREAMING, 3: GLOBAL}


def spans_for(mode: str, seq_len: int, chunk: int = 2048, origin: int = 0,
              chunks: Sequence[int] = (), local_tokens: int = 512, sink_tokens: int = 4,
              window: int = 1024) -> List[Tuple[int, int, bool]]:
    """``(start, end, round_out)`` ranges for one sequence in one mode."""
    if mode == GLOBAL:
        return [(0, seq_len, True)]
    if mode == FOCUS:
        out = []
        for c in chunks:
            start = origin + int(c) * chunk
            out.append((start, start + chunk, True))
        return out
    if mode == LOCAL:
        return [(seq_len - local_tokens, seq_len, True)]
    if mode == STREAMING:
        return [(0, sink_tokens, False), (seq_len - window, seq_len, False)]
    raise ValueError("unknown mode %r" % (mode,))


def pack(span_lists: Sequence[Sequence[Tuple[int, int, bool]]], device="cuda", max_spans: int = 0):
    """Pack per-sequence span lists into (spans int32 [B][S][2], counts int32 [B],
    round uint8 [B][S]) tensors for ``select_blocks_spans``."""
    B = len(span_lists)
    S = max([max_spans] + [len(s) for s in span_lists] + [1])
    spans = torch.zeros((B, S, 2), dtype=torch.int32)
    rnd = torch.zeros((B, S), dtype=torch.uint8)
    cnt = torch.zeros((B,), dtype=torch.int32)
    for b, lst in enumerate(span_lists):
        cnt[b] = len(lst)
        for i, (s0, s1, r) in enumerate(lst):
            spans[b, i, 0], spans[b, i, 1], rnd[b, i] = s0, s1, int(bool(r))
    return spans.to(device), cnt.to(device), rnd.to(device)
