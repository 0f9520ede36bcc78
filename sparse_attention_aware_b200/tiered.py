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

from . import _lib, api
from .cache import PagedCache

_CAPACITY = 7   # SA_ERR_CAPACITY


def span_page_ranges(spans: Sequence[Tuple[int, int, bool]], seq_len: int,
                     page_size: int) -> List[Tuple[int, int]]:
    """The pages ``span_pages`` lists, as ascending disjoint ranges [lo, hi)."""
    iv = []
    for a, b, _ in spans:
        a, b = max(a, 0), min(b, seq_len)
        if a < b:
            iv.append((a // page_size, (b - 1) // page_size + 1))
    if not iv:
        return []
    iv.sort()
    out: List[Tuple[int, int]] = []
    lo, hi = iv[0]
    for x, y in iv[1:]:
        if x > hi:
            out.append((lo, hi))
            lo, hi = x, y
        elif y > hi:
            hi = y
    out.append((lo, hi))
    return out


def span_pages(spans: Sequence[Tuple[int, int, bool]], seq_len: int, page_size: int) -> List[int]:
    """Logical pages a step reads for one sequence's span list: every page a
    span touches after clipping to [0, seq_len) (rounding a span out to page
    edges does not change the pages it touches), ascending, each once."""
    return [p for lo, hi in span_page_ranges(spans, seq_len, page_size) for p in range(lo, hi)]


class SlotMap:
    """Host bookkeeping of which host pages sit in which device slots (no GPU).

    ``plan(wanted)`` maps the pages a step reads: resident pages are hits;
    missing pages take free slots first, then the least recently used slots
    whose pages neither this step nor the step still in flight reads (by
    default the previous ``plan``'s pages).  It returns the (host page, slot)
    fetches and raises if the pool cannot hold the step.  The planning itself
    is ``sa_tier_plan`` in libsa (host code), over this object's arrays."""

    def __init__(self, host_pages: int, slots: int):
        if slots <= 0:
            raise ValueError("need at least one device slot")
        self.slots = slots
        self.slot_of = np.full(host_pages, -1, dtype=np.int32)   # host page -> slot
        self.page_in = np.full(slots, -1, dtype=np.int32)        # slot -> host page
        self.last_use = np.full(slots, -1, dtype=np.int64)
        self.tick = 0
        self.prev = np.zeros(0, dtype=np.int32)
        self.evicted: List[int] = []   # host pages the last plan evicted
        self.stats = {"hits": 0, "misses": 0}
        self._pairs = np.zeros((slots, 2), dtype=np.int32)
        self._ev = np.zeros(slots, dtype=np.int32)
        self._counts = np.zeros(4, dtype=np.int32)
        self._scratch = np.zeros(int(_lib.load().sa_tier_plan_scratch_ints(host_pages, slots)), dtype=np.int32)
        # the state arrays never move: their addresses once
        self._ptrs = tuple(x.ctypes.data for x in (self.slot_of, self.page_in, self.last_use, self._pairs,
                                                     self._ev, self._counts, self._scratch))

    def plan_array(self, wanted, in_flight: Optional[Set[int]] = None) -> np.ndarray:
        """``plan`` returning the fetches as an int32 array [n][2] (a view,
        valid until the next call)."""
        w = np.ascontiguousarray(np.asarray(wanted).ravel(), dtype=np.int32)
        keep = self.prev if in_flight is None else np.asarray(sorted(in_flight), dtype=np.int32)
        keep = np.ascontiguousarray(keep, dtype=np.int32)
        self.tick += 1
        ps, pp, pl, pa, pe, pc, px = self._ptrs
        st = _lib.load().sa_tier_plan(ps, len(self.slot_of), pp, pl, self.slots, self.tick,
                                      w.__array_interface__["data"][0], len(w),
                                      keep.__array_interface__["data"][0], len(keep), pa, pe, pc,
                                      px, len(self._scratch))
        if st == _CAPACITY:
            raise RuntimeError("the pages of this step (%d distinct) and of the step in flight do not fit the "
                               "device pool of %d slots" % (len(np.unique(w)), self.slots))
        if st != _lib.SA_OK:
            raise ValueError("sa_tier_plan: %s" % _lib.STATUS_NAMES.get(st, st))
        n, m, hits, _ = (int(x) for x in self._counts)
        self.stats["hits"] += hits
        self.stats["misses"] += n
        self.evicted = self._ev[:m].tolist()
        self.prev = w
        return self._pairs[:n]

    def plan(self, wanted: Sequence[int], in_flight: Optional[Set[int]] = None) -> List[Tuple[int, int]]:
        return [(int(p), int(s)) for p, s in self.plan_array(wanted, in_flight)]


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
        lens = [len(p) for p in need]
        lp = np.fromiter((x for pages in need for x in pages), dtype=np.int64, count=sum(lens))
        b = np.repeat(np.arange(len(need), dtype=np.int64), lens)
        return self.host_pt[b, lp]

    def prepare_spans(self, span_lists: Sequence[Sequence[Tuple[int, int, bool]]], seq_lens: Sequence[int],
                      compute_stream: Optional[torch.cuda.Stream] = None) -> int:
        """``prepare`` for the pages of per-sequence span lists (the pages
        ``span_pages(span_lists[b], seq_lens[b], P)`` names), mapped through
        the host page table range by range."""
        parts = [self.host_pt[b, lo:hi] for b, (spans, n) in enumerate(zip(span_lists, seq_lens))
                 for lo, hi in span_page_ranges(spans, n, self.P)]
        wanted = np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)
        return self._prepare_pages(wanted, compute_stream, seq_lens)

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
        return self._prepare_pages(self.host_pages_of(need), compute_stream, seq_lens)

    def _prepare_pages(self, wanted: np.ndarray, compute_stream, seq_lens) -> int:
        compute_stream = compute_stream or torch.cuda.current_stream(self.device)
        # the step queued just before this call may still be running and its
        # pages are kept; older steps must be done before a slot is reused
        mark = torch.cuda.Event()
        mark.record(compute_stream)
        pairs = self.map.plan_array(wanted)
        changed = len(pairs) > 0
        if self.map.evicted:
            ev = np.asarray(self.map.evicted)
            self.pt[self.where_b[ev], self.where_lp[ev]] = -1
        if changed:
            self.pt[self.where_b[pairs[:, 0]], self.where_lp[pairs[:, 0]]] = pairs[:, 1]
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
            if changed:
                n = len(pairs)
                hb = self.pflip
                self.pflip ^= 1
                if self.pairs_free[hb] is not None:
                    self.pairs_free[hb].synchronize()     # its copy two fetches ago is done
                self.pairs_host[hb].numpy()[:n] = pairs
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
