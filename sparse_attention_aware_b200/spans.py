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
    import numpy as np
    B = len(span_lists)
    S = max([max_spans] + [len(s) for s in span_lists] + [1])
    spans = np.zeros((B, S, 2), dtype=np.int32)
    rnd = np.zeros((B, S), dtype=np.uint8)
    cnt = np.zeros((B,), dtype=np.int32)
    for b, lst in enumerate(span_lists):
        n = len(lst)
        cnt[b] = n
        if n:
            spans[b, :n] = [(s0, s1) for s0, s1, _ in lst]
            rnd[b, :n] = [1 if r else 0 for _, _, r in lst]
    return (torch.from_numpy(spans).to(device), torch.from_numpy(cnt).to(device),
            torch.from_numpy(rnd).to(device))
