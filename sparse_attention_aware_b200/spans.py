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


class SpanPacker:
    """``pack`` for a serving loop: the span lists of a step are written into
    one of ``depth`` pinned host buffers and copied to fixed device tensors
    with non-blocking copies on the caller's stream, so the host does not wait
    for the GPU (a copy from pageable memory would wait for the stream).  A
    host buffer is rewritten only after the copy that last read it has
    completed; the device tensors are rewritten by a copy queued on the same
    stream as the kernels that read them, so stream order protects them."""

    def __init__(self, batch: int, max_spans: int, device, depth: int = 2):
        import numpy as np
        self.B, self.S = batch, max(1, max_spans)
        self.device = torch.device(device)
        self.host = [(torch.zeros((batch, self.S, 2), dtype=torch.int32).pin_memory(),
                      torch.zeros((batch,), dtype=torch.int32).pin_memory(),
                      torch.zeros((batch, self.S), dtype=torch.uint8).pin_memory()) for _ in range(depth)]
        self.done = [None] * depth
        self.dev = (torch.zeros((batch, self.S, 2), dtype=torch.int32, device=self.device),
                    torch.zeros((batch,), dtype=torch.int32, device=self.device),
                    torch.zeros((batch, self.S), dtype=torch.uint8, device=self.device))
        self.i = 0
        self._np = np

    def pack(self, span_lists: Sequence[Sequence[Tuple[int, int, bool]]], stream=None):
        """Device (spans, counts, round) for ``span_lists`` (one list per
        sequence, at most ``max_spans`` spans each)."""
        if len(span_lists) != self.B:
            raise ValueError("need one span list per sequence (%d)" % self.B)
        k = self.i % len(self.host)
        self.i += 1
        if self.done[k] is not None:
            self.done[k].synchronize()
        hs, hc, hr = self.host[k]
        ns, nc, nr = hs.numpy(), hc.numpy(), hr.numpy()
        ns[...] = 0
        nc[...] = 0
        nr[...] = 0
        for b, lst in enumerate(span_lists):
            n = len(lst)
            if n > self.S:
                raise ValueError("sequence %d has %d spans, the packer holds %d" % (b, n, self.S))
            nc[b] = n
            for j, (s0, s1, r) in enumerate(lst):
                ns[b, j, 0], ns[b, j, 1], nr[b, j] = s0, s1, 1 if r else 0
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.stream(s):
            for d, h in zip(self.dev, self.host[k]):
                d.copy_(h, non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(s)
        self.done[k] = ev
        return self.dev
