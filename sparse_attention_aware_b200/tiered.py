"""Tiered KV: a host-memory tier behind a fixed pool of device page slots.

A DA step only hides context; it deletes none.  So the KV pages no step is
reading can wait in an outer tier and be fetched back, alongside decoding,
when a declaration names them again ("语言模型能自己决定该看哪里吗？", on
moving ignored KV to outer memory), and the KV cache becomes tiered storage
with the focus regions loaded on demand ("百万上下文，模型终于会挑重点了",
"对百万上下文产品意味着什么").

``TieredKV`` keeps every page of a static paged cache in pinned host memory
(the master copy) and ``slots`` device page slots.  Before a step it is told
which logical pages the step reads (from the span lists of the DA state
machine, or any page set); it maps resident pages, picks free or
least-recently-used slots for the missing ones (never a slot that a step
still in flight reads), gathers them with one ``sa_fetch_pages`` launch on
its copy stream, and publishes a device page table (logical page -> slot;
-1 for pages not resident, so that a read of one is recorded as a device
fault, not served from a stale slot).  The selection and decode kernels read
``cache`` exactly like a fully resident cache.
"""
from __future__ import annotations

from typing import Iterable, List, Optional, Sequence, Set, Tuple

import numpy as np
import torch

from . import api
from .cache import PagedCache


def span_pages(spans: Sequence[Tuple[int, int, bool]], seq_len: int, page_size: int) -> List[int]:
    """Logical pages a step reads for one sequence's span list: every page a
    span touches after clipping to [0, seq_len) (rounding a span out to page
    edges does not change the pages it touches), ascending."""
    parts = []
    for a, b, _ in spans:
        a, b = max(a, 0), min(b, seq_len)
        if a < b:
            parts.append(np.arange(a // page_size, (b - 1) // page_size + 1))
    if not parts:
        return []
    return np.unique(np.concatenate(parts)).tolist()


class SlotMap:
    """Host bookkeeping of which host pages sit in which device slots (no GPU).

    ``plan(wanted)`` maps the pages a step reads: resident pages are hits;
    missing pages take free slots first, then the least recently used slots
    whose pages neither this step nor the step still in flight reads (by
    default the previous ``plan``'s pages).  It returns the (host page, slot)
    fetches and raises if the pool cannot hold the step."""

    def __init__(self, host_pages: int, slots: int):
        if slots <= 0:
            raise ValueError("need at least one device slot")
        self.slots = slots
        self.slot_of = np.full(host_pages, -1, dtype=np.int64)   # host page -> slot
        self.page_in = np.full(slots, -1, dtype=np.int64)        # slot -> host page
        self.last_use = np.full(slots, -1, dtype=np.int64)
        self.tick = 0
        self.prev = np.zeros(0, dtype=np.int64)
        self.evicted: List[int] = []   # host pages the last plan evicted
        self.stats = {"hits": 0, "misses": 0}

    def plan(self, wanted: Sequence[int], in_flight: Optional[Set[int]] = None) -> List[Tuple[int, int]]:
        self.tick += 1
        w = np.asarray(wanted, dtype=np.int64).ravel()
        _, first = np.unique(w, return_index=True)
        w = w[np.sort(first)]                      # distinct, in first-occurrence order
        if len(w) > self.slots:
            raise RuntimeError("step needs %d pages, the device pool has %d slots" % (len(w), self.slots))
        prev = self.prev if in_flight is None else np.asarray(sorted(in_flight), dtype=np.int64)
        keep = np.union1d(w, prev)
        slots_w = self.slot_of[w]
        hit = slots_w >= 0
        self.last_use[slots_w[hit]] = self.tick
        self.stats["hits"] += int(hit.sum())
        missing = w[~hit]
        pairs = []
        self.evicted = []
        if len(missing):
            free = np.nonzero(self.page_in < 0)[0]
            cand = free
            if len(free) < len(missing):
                used = np.nonzero((self.page_in >= 0) & ~np.isin(self.page_in, keep))[0]
                used = used[np.lexsort((used, self.last_use[used]))]
                cand = np.concatenate([free, used[: len(missing) - len(free)]])
            if len(cand) < len(missing):
                raise RuntimeError("not enough evictable slots: the pages of this step and of the step in "
                                   "flight exceed the device pool")
            cand = cand[: len(missing)]
            old = self.page_in[cand]
            ev = old[old >= 0]
            self.slot_of[ev] = -1
            self.evicted = ev.tolist()
            self.page_in[cand] = missing
            self.slot_of[missing] = cand
            self.last_use[cand] = self.tick
            pairs = list(zip(missing.tolist(), cand.tolist()))
            self.stats["misses"] += len(missing)
        self.prev = w
        return pairs


class TieredKV:
    def __init__(self, cache: PagedCache, slots: int, device, copy_stream: Optional[torch.cuda.Stream] = None,
                 time_fetches: bool = False):
        """``cache``: the full cache (any device); it becomes the pinned host
        tier.  ``slots``: device page slots.  With ``time_fetches`` every
        fetch launch is bracketed by CUDA events (``fetch_events``)."""
        self.device = torch.device(device)
        self.P = cache.k.shape[2]
        self.host_k = cache.k.cpu().pin_memory()
        self.host_v = cache.v.cpu().pin_memory()
        self.host_pt = cache.page_table.cpu().numpy().astype(np.int64)   # logical -> host page
        # sequence lengths, published with the page table: two device copies
        # used alternately (the step in flight keeps reading its own), each
        # filled from a pinned mirror on the copy stream
        lens0 = cache.seq_lens.to(torch.int32).cpu()
        self.dev_lens = [lens0.to(self.device), lens0.to(self.device)]
        self.lens_mirror = [lens0.clone().pin_memory() for _ in range(2)]
        self.lens_free = [None, None]
        self.lens_cur = 0
        self.map = SlotMap(self.host_k.shape[0], slots)
        shape = (slots,) + tuple(self.host_k.shape[1:])
        self.dev_k = torch.zeros(shape, dtype=torch.bfloat16, device=self.device)
        self.dev_v = torch.zeros(shape, dtype=torch.bfloat16, device=self.device)
        # where each host page sits in the logical page table (one entry each)
        self.where_b = np.zeros(self.host_k.shape[0], dtype=np.int64)
        self.where_lp = np.zeros(self.host_k.shape[0], dtype=np.int64)
        bb, ll = np.nonzero(self.host_pt >= 0)
        if len(np.unique(self.host_pt[bb, ll])) != len(bb):
            raise ValueError("a host page is referenced by more than one (sequence, logical page)")
        self.where_b[self.host_pt[bb, ll]] = bb
        self.where_lp[self.host_pt[bb, ll]] = ll
        self.pt = np.full(self.host_pt.shape, -1, dtype=np.int32)   # published table, host copy
        # two pinned mirrors, used alternately, so the host never waits for the
        # copy of the previous step's table
        self.pt_mirror = [torch.full(self.host_pt.shape, -1, dtype=torch.int32).pin_memory() for _ in range(2)]
        self.mirror_free = [None, None]
        self.flip = 0
        self.dev_pt = torch.full(self.host_pt.shape, -1, dtype=torch.int32, device=self.device)
        # (host page, slot) fetch lists: two pinned host buffers used alternately
        # (a pinned allocation per step costs milliseconds) and one device
        # buffer, rewritten on the copy stream after the previous fetch read it
        self.pairs_host = [torch.zeros((slots, 2), dtype=torch.int32).pin_memory() for _ in range(2)]
        self.pairs_free = [None, None]
        self.pflip = 0
        self.pairs_dev = torch.zeros((slots, 2), dtype=torch.int32, device=self.device)
        self.stream = copy_stream or torch.cuda.Stream(self.device)
        self.ws = api.Workspace(self.device)
        self.ready = torch.cuda.Event()
        self.ready.record(self.stream)
        self.prev_mark = None   # compute-stream work queued before the previous prepare
        self.fetched_bytes = 0
        self.time_fetches = time_fetches
        self.fetch_events = []

    @property
    def cache(self) -> PagedCache:
        """The device view: slot pools and the published page table."""
        return PagedCache(self.dev_k, self.dev_v, self.dev_pt, self.dev_lens[self.lens_cur])

    @property
    def seq_lens(self) -> torch.Tensor:
        return self.dev_lens[self.lens_cur]

    def page_bytes(self) -> int:
        return self.host_k[0].numel() * 2

    def host_pages_of(self, need: Sequence[Iterable[int]]) -> np.ndarray:
        parts = [self.host_pt[b, np.asarray(pages, dtype=np.int64)] for b, pages in enumerate(need) if len(pages)]
        return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)

    def prepare(self, need: Sequence[Iterable[int]], compute_stream: Optional[torch.cuda.Stream] = None,
                seq_lens: Optional[Sequence[int]] = None) -> int:
        """Make the logical pages ``need[b]`` of every sequence resident:
        fetch the missing ones and publish the page table on the copy stream;
        the compute stream waits for both before its next launch.  Returns the
        number of pages fetched.

        ``seq_lens`` (one per sequence) are published with the table and
        become ``cache.seq_lens`` for the step.  The span and top-k kernels clip
        what they read to these lengths, so ``need`` must be computed with the
        same ones (``span_pages(spans, seq_lens[b], P)``): a span that reaches
        past the length the host clipped to would make the device read a page
        that was never requested."""
        compute_stream = compute_stream or torch.cuda.current_stream(self.device)
        # the step queued just before this call may still be running and its
        # pages are kept; older steps must be done before a slot is reused
        mark = torch.cuda.Event()
        mark.record(compute_stream)
        pairs = self.map.plan(self.host_pages_of(need))
        changed = bool(pairs)
        if self.map.evicted:
            ev = np.asarray(self.map.evicted)
            self.pt[self.where_b[ev], self.where_lp[ev]] = -1
        if pairs:
            pa = np.asarray(pairs)
            self.pt[self.where_b[pa[:, 0]], self.where_lp[pa[:, 0]]] = pa[:, 1]
        lbuf = self.lens_cur ^ 1
        if seq_lens is not None:
            if len(seq_lens) != self.host_pt.shape[0]:
                raise ValueError("seq_lens: one length per sequence")
            if self.lens_free[lbuf] is not None:
                self.lens_free[lbuf].synchronize()
            self.lens_mirror[lbuf].numpy()[...] = np.asarray(seq_lens, dtype=np.int32)
        buf = self.flip
        if changed:
            self.flip ^= 1
            if self.mirror_free[buf] is not None:
                self.mirror_free[buf].synchronize()   # its copy two prepares ago is done
            self.pt_mirror[buf].numpy()[...] = self.pt
        with torch.cuda.stream(self.stream):
            if self.prev_mark is not None:
                self.stream.wait_event(self.prev_mark)
            if pairs:
                n = len(pairs)
                hb = self.pflip
                self.pflip ^= 1
                if self.pairs_free[hb] is not None:
                    self.pairs_free[hb].synchronize()     # its copy two fetches ago is done
                self.pairs_host[hb].numpy()[:n] = np.asarray(pairs, dtype=np.int32)
                pr = self.pairs_dev[:n]
                pr.copy_(self.pairs_host[hb][:n], non_blocking=True)
                done_p = torch.cuda.Event()
                done_p.record(self.stream)
                self.pairs_free[hb] = done_p
                if self.time_fetches:
                    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    ev[0].record(self.stream)
                api.fetch_pages(self.host_k, self.host_v, self.dev_k, self.dev_v, pr, ws=self.ws,
                                stream=self.stream)
                if self.time_fetches:
                    ev[1].record(self.stream)
                    self.fetch_events.append(ev)
                self.fetched_bytes += 2 * len(pairs) * self.page_bytes()
            if changed:
                self.dev_pt.copy_(self.pt_mirror[buf], non_blocking=True)
                done = torch.cuda.Event()
                done.record(self.stream)
                self.mirror_free[buf] = done
            if seq_lens is not None:
                # the buffer last served the step before the one in flight,
                # which prev_mark orders before this copy
                self.dev_lens[lbuf].copy_(self.lens_mirror[lbuf], non_blocking=True)
                done = torch.cuda.Event()
                done.record(self.stream)
                self.lens_free[lbuf] = done
            self.ready.record(self.stream)
        compute_stream.wait_event(self.ready)
        if seq_lens is not None:
            self.lens_cur = lbuf
        self.prev_mark = mark
        return len(pairs)
