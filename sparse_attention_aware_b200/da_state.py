"""Host-side DA state machine: from the model's output stream to span lists.

The DA state machine runs beside the inference engine, watches the tokens the
model emits for mode declarations, and sets, for the next decode step, which
KV positions the step may read, at chunk granularity ("语言模型能自己决定该看
哪里吗？", the DA state machine / vLLM section).  The modes are ``<global>``
(the whole context), ``<focus>`` (declared regions) and ``<local>`` (recent
output only), and the model switches between them during generation
("百万上下文，模型终于会挑重点了", section "三种模式，背后是三种推理状态").
The same page ("但它不是免费的午餐") asks a reliable engine for fallbacks:
a periodic global check, forced ``<global>`` for high-risk tasks, a minimum
neighbourhood around focus regions, and a wider read range when the model is
not confident.  All four are parameters here.

The output of a step is a list of ``(start, end, round_out)`` token spans per
sequence, the input of ``select_blocks_spans`` (which rounds DA spans out to
page edges, clips them to the sequence, merges overlaps and lays the result
out per page on the GPU).

Readings where the pages leave a step open (no model, so the tag stream is
scripted; the token ids below are this module's, not a tokenizer's):

* A focus declaration is ``FOCUS_OPEN, CHUNK(c1), CHUNK(c2), ..., FOCUS_CLOSE``;
  chunk ``c`` is the magic chunk ``[origin + c*chunk, origin + (c+1)*chunk)``
  of the prompt.  The new mode takes effect on the step after the token that
  completes the declaration (``GLOBAL``, ``LOCAL`` or ``FOCUS_CLOSE``); while
  a focus declaration is open the previous mode stays in effect.
* A focus declaration that names no chunk inside the prompt falls back to
  ``<global>``: an empty or invalid declaration must not hide the context.
* Before any declaration the mode is ``<global>``.
* ``<local>`` reads the last ``local_tokens`` (512) tokens, rounded out to
  pages like focus regions.
* Low confidence (a per-step value below ``low_conf_threshold``, supplied by
  the caller) either reads globally (``low_conf_action="global"``) or widens
  the step's regions (``"widen"``: every focus region by one chunk on each
  side, the local window fourfold).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

from . import spans as SP

Span = Tuple[int, int, bool]


@dataclasses.dataclass(frozen=True)
class DAVocab:
    """Token ids of the mode tags.  ``CHUNK(c)`` is ``chunk_base + c``."""
    global_tag: int = 1_000_001
    local_tag: int = 1_000_002
    focus_open: int = 1_000_003
    focus_close: int = 1_000_004
    chunk_base: int = 2_000_000
    max_chunks: int = 1 << 20

    def chunk_id(self, token: int) -> Optional[int]:
        c = token - self.chunk_base
        return c if 0 <= c < self.max_chunks else None


@dataclasses.dataclass(frozen=True)
class DAFallbacks:
    """Safety fallbacks ("但它不是免费的午餐").  0 / False switch one off."""
    periodic_global: int = 0          # every n-th step (n, 2n, ...) reads globally
    force_global: bool = False        # high-risk task: every step reads globally
    focus_margin: int = 0             # tokens added on each side of every focus region
    low_conf_threshold: float = 0.0   # confidence below this widens the step
    low_conf_action: str = "global"   # "global" or "widen"


class DAStateMachine:
    """State of one sequence: the mode in effect and a pending declaration."""

    def __init__(self, prompt_len: int, chunk: int = 2048, origin: int = 0, local_tokens: int = 512,
                 vocab: DAVocab = DAVocab(), fallbacks: DAFallbacks = DAFallbacks()):
        if prompt_len < 0 or chunk <= 0 or local_tokens <= 0:
            raise ValueError("bad DA state machine parameters")
        if fallbacks.low_conf_action not in ("global", "widen"):
            raise ValueError("low_conf_action must be 'global' or 'widen'")
        self.prompt_len = prompt_len
        self.chunk = chunk
        self.origin = origin
        self.local_tokens = local_tokens
        self.vocab = vocab
        self.fb = fallbacks
        self.mode = SP.GLOBAL
        self.focus: Tuple[int, ...] = ()
        self._open: Optional[List[int]] = None   # chunk ids of an open focus declaration
        self.steps = 0

    # -- stream ---------------------------------------------------------------
    def _valid_chunks(self, ids: Sequence[int]) -> Tuple[int, ...]:
        """Distinct declared chunks that meet the prompt, in declaration order."""
        out = []
        for c in ids:
            a = self.origin + c * self.chunk
            if a < self.prompt_len and a + self.chunk > 0 and c not in out:
                out.append(c)
        return tuple(out)

    def observe(self, token: int) -> None:
        """Feed the token the model emitted at this step."""
        v = self.vocab
        if self._open is not None:
            if token == v.focus_close:
                chunks = self._valid_chunks(self._open)
                self._open = None
                if chunks:
                    self.mode, self.focus = SP.FOCUS, chunks
                else:
                    self.mode, self.focus = SP.GLOBAL, ()
                return
            c = v.chunk_id(token)
            if c is not None:
                self._open.append(c)
                return
            # any other tag aborts the open declaration and is handled below
            if token not in (v.global_tag, v.local_tag, v.focus_open):
                return
            self._open = None
        if token == v.global_tag:
            self.mode, self.focus = SP.GLOBAL, ()
        elif token == v.local_tag:
            self.mode, self.focus = SP.LOCAL, ()
        elif token == v.focus_open:
            self._open = []

    # -- next step --------------------------------------------------------------
    def next_spans(self, seq_len: int, confidence: float = 1.0) -> List[Span]:
        """Spans the next decode step may read (the context is ``seq_len`` long,
        prompt and generated tokens); advances the step counter."""
        self.steps += 1
        fb = self.fb
        mode = self.mode
        if fb.force_global or (fb.periodic_global > 0 and self.steps % fb.periodic_global == 0):
            mode = SP.GLOBAL
        widen = confidence < fb.low_conf_threshold
        if widen and fb.low_conf_action == "global":
            mode = SP.GLOBAL
        if mode == SP.GLOBAL:
            return SP.spans_for(SP.GLOBAL, seq_len)
        if mode == SP.LOCAL:
            local = self.local_tokens * (4 if widen else 1)
            return SP.spans_for(SP.LOCAL, seq_len, local_tokens=local)
        chunks = self.focus
        if widen:
            grown = []
            for c in chunks:
                for d in (c - 1, c, c + 1):
                    if d not in grown:
                        grown.append(d)
            chunks = self._valid_chunks(grown)
        out = []
        for a, b, r in SP.spans_for(SP.FOCUS, seq_len, self.chunk, self.origin, chunks):
            out.append((a - fb.focus_margin, b + fb.focus_margin, r))
        return out


class DABatch:
    """One state machine per sequence of a decode batch."""

    def __init__(self, prompt_lens: Sequence[int], **kw):
        self.machines = [DAStateMachine(L, **kw) for L in prompt_lens]

    def step(self, tokens: Sequence[int], seq_lens: Sequence[int], confidences: Optional[Sequence[float]] = None,
             device="cuda", max_spans: int = 0):
        """Feed each sequence's emitted token, then return the packed span
        tensors ``(spans, counts, round)`` of the next step."""
        if len(tokens) != len(self.machines) or len(seq_lens) != len(self.machines):
            raise ValueError("one token and one length per sequence")
        conf = confidences if confidences is not None else [1.0] * len(self.machines)
        lists = []
        for m, t, L, c in zip(self.machines, tokens, seq_lens, conf):
            m.observe(int(t))
            lists.append(m.next_spans(int(L), float(c)))
        return SP.pack(lists, device, max_spans=max_spans)
