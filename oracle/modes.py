"""Oracle-side reading of the decode modes as token spans -- TEST INFRASTRUCTURE.

Written independently of the product's span builder.  Each mode becomes a list
of ``(start, end, round_out)`` token spans over a sequence of length ``L``:

* DA ``<focus>`` ("百万上下文，模型终于会挑重点了", section "三种模式"; and
  "语言模型能自己决定该看哪里吗？", on magic chunks of about 2048 tokens and
  block-aligned masks): the declared chunks ``[o + c*C, o + (c+1)*C)``, each
  rounded out to page edges.
* DA ``<local>``: only recent tokens; read here as the last ``local_window``
  (512) tokens, rounded out like focus.
* DA ``<global>``: the whole context ``[0, L)``.
* LoZA streaming window ("稀疏注意力机制创新…", section "二、ZigZag架构"): a
  fixed 1024-token window over the most recent tokens, plus 4 sink tokens at
  the start, token-exact (not rounded).
"""
from __future__ import annotations

FOCUS, LOCAL, STREAM, GLOBAL = 0, 1, 2, 3


def mode_spans(mode: int, L: int, chunk: int = 2048, origin: int = 0, focus_chunks=(),
               local_window: int = 512, sinks: int = 4, window: int = 1024):
    if mode == FOCUS:
        return [(origin + c * chunk, origin + (c + 1) * chunk, True) for c in focus_chunks]
    if mode == LOCAL:
        return [(L - local_window, L, True)]
    if mode == GLOBAL:
        return [(0, L, True)]
    if mode == STREAM:
        return [(0, sinks, False), (L - window, L, False)]
    raise ValueError(mode)
