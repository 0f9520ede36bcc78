"""Python binding of libsa: the four entry points with the C ABI's names.

Argument marshalling only: tensors are passed to the C library as raw device
pointers on torch's current stream, outputs and workspaces are allocated with
torch when the caller does not pass them.  Every step of the computation runs
in libsa's CUDA kernels; if the library is missing, ``_lib.load`` raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import functools
import math
from typing import Optional, Sequence

import torch

from . import _lib as L


class SAError(RuntimeError):
    def __init__(self, status: int, where: str, detail=None):
        self.status = status
        self.detail = detail
        msg = "%s: %s" % (where, L.load().sa_status_string(status).decode())
        if detail is not None:
            msg += " (check %d, value %d)" % (detail[1], detail[2])
        super().__init__(msg)


def _check(status: int, where: str):
    if status != L.SA_OK:
        raise SAError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _on_call_stream(fn):
    """When an entry point is given ``stream=``, the tensors it makes itself
    (contiguous copies of inputs, threshold tensors, default outputs, a
    growing workspace) are made on that stream, so that they are ordered
    before the kernels that read them and the caching allocator does not hand
    their memory out again while those kernels run.  Without ``stream=`` the
    call runs on torch's current stream as before."""
    @functools.wraps(fn)
    def call(*args, **kw):
        s = kw.get("stream")
        if s is None:
            return fn(*args, **kw)
        with torch.cuda.stream(s):
            return fn(*args, **kw)
    return call


def kv_struct(cache, device=None) -> L.KVCacheS:
    """``cache``: any object with k, v, page_table, seq_lens tensors on the GPU
    (k/v bf16 [num_pages][Hkv][P][d], page_table int32 [B][max_pages],
    seq_lens int32 [B]).  ``device``: when given, every cache tensor must be on
    it (the device of the call's queries).  Raises ValueError otherwise."""
    k, v = cache.k, cache.v
    pt, sl = cache.page_table, cache.seq_lens
    if k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise ValueError("KV cache: k and v must be bf16, got %s / %s" % (k.dtype, v.dtype))
    if k.dim() != 4 or k.shape != v.shape or not k.is_contiguous() or not v.is_contiguous():
        raise ValueError("KV cache: k and v must be contiguous [num_pages][Hkv][P][d] tensors of one shape")
    if pt.dtype != torch.int32 or pt.dim() != 2 or not pt.is_contiguous():
        raise ValueError("KV cache: page_table must be a contiguous int32 [B][max_pages] tensor")
    if sl.dtype != torch.int32 or tuple(sl.shape) != (pt.shape[0],) or not sl.is_contiguous():
        raise ValueError("KV cache: seq_lens must be a contiguous int32 [B] tensor, B = %d" % pt.shape[0])
    devs = {t.device for t in (k, v, pt, sl)}
    if device is not None:
        devs.add(torch.device(device))
    if len(devs) != 1:
        raise ValueError("KV cache: k, v, page_table, seq_lens and the queries must be on one device, got %s"
                         % sorted(str(d) for d in devs))
    return L.KVCacheS(k.data_ptr(), v.data_ptr(), pt.data_ptr(), sl.data_ptr(), pt.shape[0], k.shape[1],
                      k.shape[3], k.shape[2], pt.shape[1], k.shape[0])


class Workspace:
    """A reusable, zero-initialised device workspace (grows on demand).

    A workspace belongs to one stream at a time: calls that share it must be
    ordered on the GPU (same stream, or events between streams), since every
    call rewrites its status header and scratch.  When it grows, the old
    buffer is released with record_stream() for every stream it was handed
    to, so the caching allocator does not reuse that memory while a kernel
    launched on one of those streams may still read it."""

    def __init__(self, device=None):
        self.device = device
        self.buf: Optional[torch.Tensor] = None
        self._streams = []

    def get(self, nbytes: int, stream=None) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes:
            n = max(nbytes, 256)
            old = self.buf
            self.buf = torch.zeros(n + 256, dtype=torch.uint8, device=self.device or "cuda")
            if old is not None:
                for s in self._streams:
                    old.record_stream(s)
            self._streams = []
        if self.buf.device.type == "cuda":
            s = stream if stream is not None else torch.cuda.current_stream(self.buf.device)
            if all(s != x for x in self._streams):
                self._streams.append(s)
        return self.buf

    def aligned(self, nbytes: int, stream=None):
        buf = self.get(nbytes, stream)
        base = buf.data_ptr()
        off = (-base) % 256
        return ctypes.c_void_p(base + off), buf.numel() - off

    def status(self, stream=None):
        """Synchronise and return (status, detail) recorded by kernels (then cleared)."""
        if self.buf is None:
            return 0, (0, 0, 0)
        ptr, _ = self.aligned(0, stream)
        det = (L.c_i32 * 3)()
        st = L.load().sa_read_device_status(ptr, _stream(stream), det)
        return st, tuple(det)

    def raise_on_fault(self, where="device", stream=None):
        st, det = self.status(stream)
        if st != 0:
            raise SAError(st, where, det)


_default_ws = {}


def _ws(ws: Optional[Workspace], device, stream=None) -> Workspace:
    """The caller's workspace, else a default one per (device, stream), so
    that calls on different streams never share scratch."""
    if ws is not None:
        return ws
    dev = torch.device(device)
    if stream is not None:
        sid = int(stream.cuda_stream)
    elif dev.type == "cuda":
        sid = int(torch.cuda.current_stream(dev).cuda_stream)
    else:
        sid = 0
    key = (str(dev), sid)
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key]


def workspace_bytes(op: int, cache, num_q_heads=0, k=0, num_splits=0, num_tokens=0,
                    block_args: Optional[L.BlockSelectArgsS] = None) -> int:
    kv = kv_struct(cache)
    q = L.WsQueryS(num_q_heads, k, num_splits, num_tokens,
                   ctypes.pointer(block_args) if block_args is not None else None)
    n = L.load().sa_workspace_bytes(op, ctypes.byref(kv), ctypes.byref(q))
    if n == 0:
        raise SAError(1, "sa_workspace_bytes")
    return n


def _need(t: torch.Tensor, shape, dtype, device, what: str) -> None:
    """A caller-provided output (or index) tensor must have exactly the layout
    the library writes: shape, dtype, contiguity and device."""
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous() or t.device != device:
        raise ValueError("%s: need a contiguous %s tensor of shape %s on %s, got %s %s on %s"
                         % (what, dtype, tuple(shape), device, t.dtype, tuple(t.shape), t.device))


def _bf16_q(q: torch.Tensor, what: str) -> torch.Tensor:
    if q.dtype != torch.bfloat16:
        raise TypeError("%s: q must be bf16, got %s" % (what, q.dtype))
    return q.contiguous()


def _qdtype(q: torch.Tensor) -> int:
    if q.dtype == torch.float32:
        return L.DTYPE_F32
    if q.dtype == torch.bfloat16:
        return L.DTYPE_BF16
    raise TypeError("q must be fp32 or bf16")


# --------------------------------------------------------------------------
# selections
# --------------------------------------------------------------------------
@dataclasses.dataclass
class TokenSelection:
    idx: torch.Tensor     # int32 [B][Hq][k_cap]
    count: torch.Tensor   # int32 [B][Hq]

    def struct(self) -> L.SelectionS:
        return L.SelectionS(L.SEL_TOKENS, self.idx.data_ptr(), self.count.data_ptr(), self.idx.shape[-1],
                            None, None, 0)


@dataclasses.dataclass
class BlockSelection:
    blocks: torch.Tensor        # int32 [B][max_blocks][4]
    block_counts: torch.Tensor  # int32 [B]

    def struct(self) -> L.SelectionS:
        return L.SelectionS(L.SEL_BLOCKS, None, None, 0, self.blocks.data_ptr(),
                            self.block_counts.data_ptr(), self.blocks.shape[1])


@dataclasses.dataclass
class BlockCSR:
    row_ptr: torch.Tensor   # int32 [Hq*nQB + 1]
    cols: torch.Tensor      # int32 [nnz_capacity]
    tau: torch.Tensor       # fp32 [2][Hq] thresholds applied
    num_q_heads: int
    num_q_blocks: int


def _check_selection(sel, B: int, Hq: int, device) -> None:
    """The selection tensors a decode reads must have the layout the kernels
    index: token lists idx int32 [B][Hq][k_cap] and count int32 [B][Hq];
    block lists blocks int32 [B][max_blocks][4] and block_counts int32 [B];
    contiguous, on the queries' device.  Raises ValueError otherwise."""
    if isinstance(sel, TokenSelection):
        if sel.idx.dim() != 3:
            raise ValueError("TokenSelection.idx must be int32 [B][Hq][k_cap], got shape %s" % (tuple(sel.idx.shape),))
        _need(sel.idx, (B, Hq, sel.idx.shape[-1]), torch.int32, device, "TokenSelection.idx")
        _need(sel.count, (B, Hq), torch.int32, device, "TokenSelection.count")
    elif isinstance(sel, BlockSelection):
        if sel.blocks.dim() != 3:
            raise ValueError("BlockSelection.blocks must be int32 [B][max_blocks][4], got shape %s"
                             % (tuple(sel.blocks.shape),))
        _need(sel.blocks, (B, sel.blocks.shape[1], 4), torch.int32, device, "BlockSelection.blocks")
        _need(sel.block_counts, (B,), torch.int32, device, "BlockSelection.block_counts")
    else:
        raise TypeError("selection must be a TokenSelection or a BlockSelection, got %s" % type(sel).__name__)


# --------------------------------------------------------------------------
# entry points
# --------------------------------------------------------------------------
@_on_call_stream
def select_topk(cache, q: torch.Tensor, k: int, idx: Optional[torch.Tensor] = None,
                count: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None,
                stream=None) -> TokenSelection:
    """Anchor-layer exact top-k per query head (``sa_select_topk``)."""
    B, Hq, d = q.shape
    dev = q.device
    if idx is None:
        idx = torch.empty((B, Hq, k), dtype=torch.int32, device=dev)
    _need(idx, (B, Hq, k), torch.int32, dev, "select_topk idx")
    if count is None:
        count = torch.empty((B, Hq), dtype=torch.int32, device=dev)
    _need(count, (B, Hq), torch.int32, dev, "select_topk count")
    kv = kv_struct(cache, dev)
    w = _ws(ws, dev, stream)
    wp, wn = w.aligned(workspace_bytes(L.OP_SELECT_TOPK, cache, num_q_heads=Hq, k=k), stream)
    _check(L.load().sa_select_topk(ctypes.byref(kv), _ptr(q.contiguous()), _qdtype(q), Hq, k, _ptr(idx),
                                   _ptr(count), wp, wn, _stream(stream)), "sa_select_topk")
    return TokenSelection(idx, count)


@_on_call_stream
def sparse_decode_attn(cache, q: torch.Tensor, sel, scale: Optional[float] = None, num_splits: int = 1,
                       out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                       want_lse: bool = True, ws: Optional[Workspace] = None, stream=None):
    """Split-KV sparse decode + combine (``sa_sparse_decode_attn``).  Returns (out bf16, lse fp32)."""
    B, Hq, d = q.shape
    dev = q.device
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)
    _need(out, (B, Hq, d), torch.bfloat16, dev, "sparse_decode_attn out")
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    if lse is not None:
        _need(lse, (B, Hq), torch.float32, dev, "sparse_decode_attn lse")
    kv = kv_struct(cache, dev)
    _check_selection(sel, B, Hq, dev)
    s = sel.struct()
    w = _ws(ws, dev, stream)
    wp, wn = w.aligned(workspace_bytes(L.OP_DECODE, cache, num_q_heads=Hq, num_splits=num_splits), stream)
    _check(L.load().sa_sparse_decode_attn(ctypes.byref(kv), _ptr(q.contiguous()), _qdtype(q), Hq,
                                          ctypes.byref(s), scale, num_splits, _ptr(out), _ptr(lse), wp, wn,
                                          _stream(stream)), "sa_sparse_decode_attn")
    return out, lse


@_on_call_stream
def check_bounded_wait(timeout_s: float, device=None, ws: Optional[Workspace] = None, stream=None) -> None:
    """Enqueue the bounded-wait diagnostic (``sa_check_bounded_wait``): a wait
    on an mbarrier that nothing arrives on gives up after ``timeout_s`` and
    records SA_ERR_TIMEOUT in the workspace, which ``ws.status()`` then reads."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    w = _ws(ws, dev, stream)
    wp, wn = w.aligned(256, stream)
    _check(L.load().sa_check_bounded_wait(int(timeout_s * 1e9), wp, wn, _stream(stream)), "sa_check_bounded_wait")


@_on_call_stream
def fetch_pages(host_k: torch.Tensor, host_v: torch.Tensor, dev_k: torch.Tensor, dev_v: torch.Tensor,
                pairs: torch.Tensor, ws: Optional[Workspace] = None, stream=None) -> None:
    """Copy host-tier pages into device page slots (``sa_fetch_pages``).
    host_k/host_v: pinned CPU tensors [host_pages][Hkv][P][d] bf16; dev_k/dev_v:
    device pools [slots][Hkv][P][d]; pairs: device int32 [n][2] {host page, slot}."""
    if not (host_k.is_pinned() and host_v.is_pinned()):
        raise ValueError("the host tier must be pinned memory")
    if host_k.shape[1:] != dev_k.shape[1:] or host_v.shape != host_k.shape or dev_v.shape != dev_k.shape:
        raise ValueError("host tier and device pool pages differ in shape")
    if host_k.dtype != torch.bfloat16 or dev_k.dtype != torch.bfloat16 or host_v.dtype != torch.bfloat16 \
            or dev_v.dtype != torch.bfloat16:
        raise ValueError("KV pages are bf16")
    if pairs.dtype != torch.int32 or pairs.dim() != 2 or pairs.shape[1] != 2 or not pairs.is_contiguous():
        raise ValueError("pairs must be a contiguous int32 [n][2] tensor")
    page_bytes = host_k[0].numel() * 2 if host_k.shape[0] else dev_k[0].numel() * 2
    w = _ws(ws, dev_k.device, stream)
    wp, wn = w.aligned(256, stream)
    _check(L.load().sa_fetch_pages(host_k.data_ptr(), host_v.data_ptr(), dev_k.data_ptr(), dev_v.data_ptr(),
                                   pairs.data_ptr(), pairs.shape[0], host_k.shape[0], dev_k.shape[0], page_bytes,
                                   wp, wn, _stream(stream)), "sa_fetch_pages")


@_on_call_stream
def select_blocks_spans(cache, spans: torch.Tensor, span_counts: torch.Tensor, span_round: torch.Tensor,
                        max_blocks: Optional[int] = None, out: Optional[BlockSelection] = None,
                        ws: Optional[Workspace] = None, stream=None) -> BlockSelection:
    """Span masks -> page-segment block list (``sa_select_blocks``, mode SPANS).
    spans int32 [B][max_spans][2], span_counts int32 [B], span_round uint8 [B][max_spans]."""
    B = cache.page_table.shape[0]
    dev = spans.device
    if out is None:
        mb = max_blocks if max_blocks is not None else cache.page_table.shape[1] + spans.shape[1]
        out = BlockSelection(torch.empty((B, mb, 4), dtype=torch.int32, device=dev),
                             torch.empty((B,), dtype=torch.int32, device=dev))
    _need(out.blocks, (B, out.blocks.shape[1], 4), torch.int32, dev, "select_blocks_spans out.blocks")
    _need(out.block_counts, (B,), torch.int32, dev, "select_blocks_spans out.block_counts")
    S = spans.shape[1]
    _need(spans, (B, S, 2), torch.int32, dev, "select_blocks_spans spans")
    _need(span_counts, (B,), torch.int32, dev, "select_blocks_spans span_counts")
    if span_round.dtype == torch.bool:
        span_round = span_round.to(torch.uint8)
    _need(span_round, (B, S), torch.uint8, dev, "select_blocks_spans span_round")
    kv = kv_struct(cache, dev)
    a = L.BlockSelectArgsS()
    a.mode = L.SEL_SPANS
    a.spans, a.span_counts, a.span_round = spans.data_ptr(), span_counts.data_ptr(), span_round.data_ptr()
    a.max_spans = spans.shape[1]
    o = L.BlockListS()
    o.blocks, o.block_counts, o.max_blocks = out.blocks.data_ptr(), out.block_counts.data_ptr(), out.blocks.shape[1]
    w = _ws(ws, dev, stream)
    wp, wn = w.aligned(workspace_bytes(L.OP_SELECT_BLOCKS, cache, block_args=a), stream)
    _check(L.load().sa_select_blocks(ctypes.byref(kv), ctypes.byref(a), ctypes.byref(o), wp, wn,
                                     _stream(stream)), "sa_select_blocks(spans)")
    return out


@_on_call_stream
def select_blocks_rbs(cache, q: torch.Tensor, block_size: int = 64, scale: Optional[float] = None,
                      tau_c=None, tau_r=None, p_c: float = 0.95, p_r: float = 0.97,
                      force_diag: bool = True, force_first: bool = True,
                      nnz_capacity: Optional[int] = None, out: Optional[BlockCSR] = None,
                      ws: Optional[Workspace] = None, stream=None) -> BlockCSR:
    """RBS two-branch block selection (``sa_select_blocks``, mode RBS).
    Explicit thresholds: tau_c / tau_r fp32 [Hq] tensors (or floats);
    otherwise quantile mode with p_c / p_r."""
    T, Hq, d = q.shape
    dev = q.device
    q = _bf16_q(q, "select_blocks_rbs")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nB = (T + block_size - 1) // block_size
    if out is None:
        cap = nnz_capacity if nnz_capacity is not None else Hq * nB * (nB + 1) // 2
        out = BlockCSR(torch.empty(Hq * nB + 1, dtype=torch.int32, device=dev),
                       torch.empty(max(cap, 1), dtype=torch.int32, device=dev),
                       torch.empty((2, Hq), dtype=torch.float32, device=dev), Hq, nB)
    _need(out.row_ptr, (Hq * nB + 1,), torch.int32, dev, "select_blocks_rbs out.row_ptr")
    _need(out.cols, (out.cols.numel(),), torch.int32, dev, "select_blocks_rbs out.cols")
    _need(out.tau, (2, Hq), torch.float32, dev, "select_blocks_rbs out.tau")
    tc = tr = None
    if tau_c is not None:
        tc = torch.as_tensor(tau_c, dtype=torch.float32, device=dev).expand(Hq).contiguous()
        tr = torch.as_tensor(tau_r, dtype=torch.float32, device=dev).expand(Hq).contiguous()
    kv = kv_struct(cache, dev)
    a = L.BlockSelectArgsS()
    a.mode = L.SEL_RBS
    a.q = q.data_ptr()
    a.num_q_heads, a.num_tokens, a.block_size, a.scale = Hq, T, block_size, scale
    a.tau_c = None if tc is None else tc.data_ptr()
    a.tau_r = None if tr is None else tr.data_ptr()
    a.p_c, a.p_r = p_c, p_r
    a.force_diag, a.force_first = int(force_diag), int(force_first)
    o = L.BlockListS()
    o.row_ptr, o.cols, o.nnz_capacity = out.row_ptr.data_ptr(), out.cols.data_ptr(), out.cols.numel()
    o.tau_out = out.tau.data_ptr()
    w = _ws(ws, dev, stream)
    wp, wn = w.aligned(workspace_bytes(L.OP_SELECT_BLOCKS, cache, block_args=a), stream)
    _check(L.load().sa_select_blocks(ctypes.byref(kv), ctypes.byref(a), ctypes.byref(o), wp, wn,
                                     _stream(stream)), "sa_select_blocks(rbs)")
    return out


@_on_call_stream
def sparse_prefill_attn(cache, q: torch.Tensor, csr: BlockCSR, scale: Optional[float] = None,
                        out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                        want_lse: bool = True, ws: Optional[Workspace] = None, stream=None):
    """Causal block-sparse prefill (``sa_sparse_prefill_attn``).  Returns (out bf16, lse fp32)."""
    T, Hq, d = q.shape
    dev = q.device
    q = _bf16_q(q, "sparse_prefill_attn")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device=dev)
    _need(out, (T, Hq, d), torch.bfloat16, dev, "sparse_prefill_attn out")
    if lse is None and want_lse:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=dev)
    if lse is not None:
        _need(lse, (T, Hq), torch.float32, dev, "sparse_prefill_attn lse")
    nQB = (T + 63) // 64
    _need(csr.row_ptr, (Hq * nQB + 1,), torch.int32, dev, "sparse_prefill_attn csr.row_ptr")
    _need(csr.cols, (csr.cols.numel(),), torch.int32, dev, "sparse_prefill_attn csr.cols")
    kv = kv_struct(cache, dev)
    c = L.BlockListS()
    c.row_ptr, c.cols, c.nnz_capacity = csr.row_ptr.data_ptr(), csr.cols.data_ptr(), csr.cols.numel()
    w = _ws(ws, dev, stream)
    wp, wn = w.aligned(workspace_bytes(L.OP_PREFILL, cache, num_q_heads=Hq, num_tokens=T), stream)
    _check(L.load().sa_sparse_prefill_attn(ctypes.byref(kv), _ptr(q), Hq, T, ctypes.byref(c), scale, 1,
                                           _ptr(out), _ptr(lse), wp, wn, _stream(stream)),
           "sa_sparse_prefill_attn")
    return out, lse
