"""CPU fp64 oracle for head-aware sparse attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it and must fail loudly when the CUDA
extension is missing.

The arithmetic lives in ``sa_oracle.c`` (plain C, fp64, built with gcc into
``liboracle.so``); this module only marshals numpy arrays through ctypes and
widens the exact stored input values (bf16 / fp32) to fp64.

Parity pins (see tests/test_oracle_*.py): every function is checked against
closed forms, brute force on tiny inputs, or a library routine (torch SDPA in
fp64).  The attention outputs themselves are "parity unpinned" by the pages:
they print no numeric worked example to reproduce.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

P_D = ctypes.POINTER(ctypes.c_double)
P_I32 = ctypes.POINTER(ctypes.c_int32)
P_I64 = ctypes.POINTER(ctypes.c_int64)
P_U8 = ctypes.POINTER(ctypes.c_uint8)
P_U16 = ctypes.POINTER(ctypes.c_uint16)


def build(force: bool = False) -> str:
    """Compile ``sa_oracle.c`` with gcc (IEEE fp64, no contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-pthread", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Cache(ctypes.Structure):
    _fields_ = [("k", P_U16), ("v", P_U16), ("page_table", P_I32), ("seq_lens", P_I32),
                ("batch", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("max_pages", ctypes.c_int32), ("num_pages", ctypes.c_int32)]


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        C = ctypes.POINTER(_Cache)
        i, l, d = ctypes.c_int, ctypes.c_long, ctypes.c_double
        L.or_default_threads.restype = ctypes.c_int
        L.or_topk_scores.argtypes = [C, P_D, i, P_D, l, i]
        L.or_select_topk.argtypes = [C, P_D, i, i, P_I32, P_I32, i]
        L.or_decode_tokens.argtypes = [C, P_D, i, P_I32, i, P_I32, d, P_D, P_D, P_I64, l, i]
        L.or_decode_tokens_split.argtypes = [C, P_D, i, P_I32, i, P_I32, d, i, P_D, P_D, P_D, P_D,
                                             P_D, i]
        L.or_decode_members.argtypes = [C, P_D, i, P_U8, l, d, P_D, P_D, P_I64, l, i]
        L.or_combine.argtypes = [i, i, P_D, P_D, P_D, P_D, P_D]
        L.or_block_stats.argtypes = [C, i, i, P_D, P_D, i]
        L.or_pool_q.argtypes = [P_U16, l, i, i, i, P_D, P_D]
        L.or_pair_scores.argtypes = [P_D, P_D, P_D, P_D, i, i, i, i, d, P_D, P_D, i]
        L.or_quantile.argtypes = [P_D, l, d]
        L.or_quantile.restype = d
        L.or_sort.argtypes = [P_D, l]
        L.or_rbs_mask.argtypes = [P_D, P_D, i, i, P_D, P_D, i, i, P_U8]
        L.or_prefill.argtypes = [C, i, P_U16, i, i, P_U8, d, P_I64, l, P_D, P_D, i]
        L.or_span_members.argtypes = [l, i, i, P_I64, P_U8, P_U8]
    return _lib


def threads() -> int:
    return int(lib().or_default_threads())


# --------------------------------------------------------------------------
# marshalling
# --------------------------------------------------------------------------
def _np(t):
    """torch tensor (any device) or numpy array -> contiguous numpy on host."""
    if hasattr(t, "detach"):
        import torch
        t = t.detach()
        if t.dtype == torch.bfloat16:
            return np.ascontiguousarray(t.cpu().view(torch.int16).numpy().view(np.uint16))
        return np.ascontiguousarray(t.cpu().numpy())
    return np.ascontiguousarray(t)


def _f64(t) -> np.ndarray:
    """Exact widening of stored values (bf16 or fp32) to fp64."""
    if hasattr(t, "detach"):
        import torch
        return np.ascontiguousarray(t.detach().cpu().to(torch.float64).numpy())
    return np.ascontiguousarray(np.asarray(t, dtype=np.float64))


def _ptr(a: np.ndarray, typ):
    return a.ctypes.data_as(typ)


class CacheView:
    """Host copy of a paged cache in the layout the C oracle reads."""

    def __init__(self, cache, v=None):
        self.k = _np(cache.k)
        self.v = _np(cache.v if v is None else v)
        assert self.k.dtype == np.uint16 and self.v.dtype == np.uint16
        self.pt = _np(cache.page_table).astype(np.int32)
        self.sl = _np(cache.seq_lens).astype(np.int32)
        nP, Hkv, P, d = self.k.shape
        self.struct = _Cache(_ptr(self.k, P_U16), _ptr(self.v, P_U16), _ptr(self.pt, P_I32),
                             _ptr(self.sl, P_I32), self.pt.shape[0], Hkv, d, P, self.pt.shape[1], nP)

    @property
    def batch(self):
        return int(self.pt.shape[0])

    @property
    def head_dim(self):
        return int(self.k.shape[3])

    @property
    def num_kv_heads(self):
        return int(self.k.shape[1])

    @property
    def max_len(self):
        return int(self.pt.shape[1] * self.k.shape[2])

    def ref(self):
        return ctypes.byref(self.struct)


def _view(cache, v=None) -> CacheView:
    return cache if isinstance(cache, CacheView) else CacheView(cache, v)


# --------------------------------------------------------------------------
# top-k (anchor layer)
# --------------------------------------------------------------------------
def topk_scores(cache, q, nthreads: int = 0) -> np.ndarray:
    """raw r[b][h][t] = q_h . k_{g(h),t} in fp64 (NaN for t >= L_b)."""
    cv = _view(cache)
    qd = _f64(q)
    B, Hq, d = qd.shape
    out = np.full((B, Hq, cv.max_len), np.nan)
    lib().or_topk_scores(cv.ref(), _ptr(qd, P_D), Hq, _ptr(out, P_D), cv.max_len, nthreads)
    return out


def select_topk(cache, q, k: int, nthreads: int = 0):
    """idx int32 [B][Hq][k] (ascending, -1 padded), count int32 [B][Hq]."""
    cv = _view(cache)
    qd = _f64(q)
    B, Hq, d = qd.shape
    idx = np.empty((B, Hq, k), dtype=np.int32)
    cnt = np.empty((B, Hq), dtype=np.int32)
    lib().or_select_topk(cv.ref(), _ptr(qd, P_D), Hq, k, _ptr(idx, P_I32), _ptr(cnt, P_I32), nthreads)
    return idx, cnt


# --------------------------------------------------------------------------
# decode attention
# --------------------------------------------------------------------------
def _rows(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, len(r)


def decode_tokens(cache, q, idx, count, scale: float, v=None, rows=None, nthreads: int = 0):
    """out [n][d], lse [n] for rows (b*Hq+h) (all if None)."""
    cv = _view(cache, v)
    qd = _f64(q)
    B, Hq, d = qd.shape
    idx = np.ascontiguousarray(_np(idx).astype(np.int32))
    cnt = np.ascontiguousarray(_np(count).astype(np.int32))
    r, n = _rows(rows)
    n = n if r is not None else B * Hq
    out = np.empty((n, d))
    lse = np.empty(n)
    lib().or_decode_tokens(cv.ref(), _ptr(qd, P_D), Hq, _ptr(idx, P_I32), idx.shape[-1],
                           _ptr(cnt, P_I32), scale, _ptr(out, P_D), _ptr(lse, P_D),
                           None if r is None else _ptr(r, P_I64), n, nthreads)
    return out, lse


def decode_tokens_split(cache, q, idx, count, scale: float, num_splits: int, v=None, nthreads=0):
    cv = _view(cache, v)
    qd = _f64(q)
    B, Hq, d = qd.shape
    idx = np.ascontiguousarray(_np(idx).astype(np.int32))
    cnt = np.ascontiguousarray(_np(count).astype(np.int32))
    n = B * Hq
    out, lse = np.empty((n, d)), np.empty(n)
    pm, pl, pa = np.empty((n, num_splits)), np.empty((n, num_splits)), np.empty((n, num_splits, d))
    lib().or_decode_tokens_split(cv.ref(), _ptr(qd, P_D), Hq, _ptr(idx, P_I32), idx.shape[-1],
                                 _ptr(cnt, P_I32), scale, num_splits, _ptr(out, P_D), _ptr(lse, P_D),
                                 _ptr(pm, P_D), _ptr(pl, P_D), _ptr(pa, P_D), nthreads)
    return out, lse, pm, pl, pa


def decode_members(cache, q, member, scale: float, v=None, rows=None, nthreads: int = 0):
    """Attention over the per-sequence token set ``member`` (u8 [B][Lmax])."""
    cv = _view(cache, v)
    qd = _f64(q)
    B, Hq, d = qd.shape
    mem = np.ascontiguousarray(np.asarray(member, dtype=np.uint8))
    r, n = _rows(rows)
    n = n if r is not None else B * Hq
    out, lse = np.empty((n, d)), np.empty(n)
    lib().or_decode_members(cv.ref(), _ptr(qd, P_D), Hq, _ptr(mem, P_U8), mem.shape[1], scale,
                            _ptr(out, P_D), _ptr(lse, P_D), None if r is None else _ptr(r, P_I64),
                            n, nthreads)
    return out, lse


def combine(m_s, l_s, acc_s):
    m_s = np.ascontiguousarray(m_s, dtype=np.float64)
    l_s = np.ascontiguousarray(l_s, dtype=np.float64)
    acc_s = np.ascontiguousarray(acc_s, dtype=np.float64)
    S, d = acc_s.shape
    out, lse = np.empty(d), np.empty(1)
    lib().or_combine(S, d, _ptr(m_s, P_D), _ptr(l_s, P_D), _ptr(acc_s, P_D), _ptr(out, P_D),
                     _ptr(lse, P_D))
    return out, float(lse[0])


# --------------------------------------------------------------------------
# RBS selection
# --------------------------------------------------------------------------
def block_stats(cache, bs: int, b: int = 0, nthreads: int = 0):
    """centroid [Hkv][nB][d], radius [Hkv][nB] over sequence ``b``."""
    cv = _view(cache)
    L = int(cv.sl[b])
    nB = (L + bs - 1) // bs
    c = np.empty((cv.num_kv_heads, nB, cv.head_dim))
    r = np.empty((cv.num_kv_heads, nB))
    lib().or_block_stats(cv.ref(), b, bs, _ptr(c, P_D), _ptr(r, P_D), nthreads)
    return c, r


def pool_q(q, bs: int):
    """qbar [Hq][nB][d], qnorm [Hq][nB] from bf16 Q [T][Hq][d]."""
    qb = _np(q)
    assert qb.dtype == np.uint16
    T, Hq, d = qb.shape
    nB = (T + bs - 1) // bs
    qbar, qn = np.empty((Hq, nB, d)), np.empty((Hq, nB))
    lib().or_pool_q(_ptr(qb, P_U16), T, Hq, d, bs, _ptr(qbar, P_D), _ptr(qn, P_D))
    return qbar, qn


def pair_scores(qbar, qnorm, centroid, radius, scale: float, nthreads: int = 0):
    """S_c, S_r [Hq][nB(nB+1)/2] over causal pairs (index i(i+1)/2 + j)."""
    qbar = np.ascontiguousarray(qbar, dtype=np.float64)
    qnorm = np.ascontiguousarray(qnorm, dtype=np.float64)
    centroid = np.ascontiguousarray(centroid, dtype=np.float64)
    radius = np.ascontiguousarray(radius, dtype=np.float64)
    Hq, nB, d = qbar.shape
    Hkv = centroid.shape[0]
    nP = nB * (nB + 1) // 2
    Sc, Sr = np.empty((Hq, nP)), np.empty((Hq, nP))
    lib().or_pair_scores(_ptr(qbar, P_D), _ptr(qnorm, P_D), _ptr(centroid, P_D), _ptr(radius, P_D),
                         Hq, Hkv, nB, d, scale, _ptr(Sc, P_D), _ptr(Sr, P_D), nthreads)
    return Sc, Sr


def quantile(x, p: float) -> float:
    x = np.ascontiguousarray(x, dtype=np.float64).ravel()
    return float(lib().or_quantile(_ptr(x, P_D), len(x), p))


def sort(x) -> np.ndarray:
    x = np.array(x, dtype=np.float64).ravel()
    lib().or_sort(_ptr(x, P_D), len(x))
    return x


def rbs_mask(Sc, Sr, tau_c, tau_r, force_diag: bool = True, force_first: bool = True):
    Sc = np.ascontiguousarray(Sc, dtype=np.float64)
    Sr = np.ascontiguousarray(Sr, dtype=np.float64)
    Hq, nP = Sc.shape
    nB = int(round((np.sqrt(8 * nP + 1) - 1) / 2))
    tc = np.ascontiguousarray(np.broadcast_to(np.asarray(tau_c, dtype=np.float64), (Hq,)))
    tr = np.ascontiguousarray(np.broadcast_to(np.asarray(tau_r, dtype=np.float64), (Hq,)))
    mask = np.empty((Hq, nP), dtype=np.uint8)
    lib().or_rbs_mask(_ptr(Sc, P_D), _ptr(Sr, P_D), Hq, nB, _ptr(tc, P_D), _ptr(tr, P_D),
                      int(force_diag), int(force_first), _ptr(mask, P_U8))
    return mask


def prefill(cache, q, bs: int, mask, scale: float, rows=None, b: int = 0, nthreads: int = 0):
    """out [n][d], lse [n] for rows (t*Hq+h) (all if None)."""
    cv = _view(cache)
    qb = _np(q)
    T, Hq, d = qb.shape
    mask = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
    r, n = _rows(rows)
    n = n if r is not None else int(cv.sl[b]) * Hq
    out, lse = np.empty((n, d)), np.empty(n)
    lib().or_prefill(cv.ref(), b, _ptr(qb, P_U16), Hq, bs, _ptr(mask, P_U8), scale,
                     None if r is None else _ptr(r, P_I64), n, _ptr(out, P_D), _ptr(lse, P_D),
                     nthreads)
    return out, lse


# --------------------------------------------------------------------------
# spans
# --------------------------------------------------------------------------
def span_members(L: int, P: int, spans: Sequence) -> np.ndarray:
    """u8 [L] membership of tokens in the union of spans ``(a, b, round_out)``."""
    n = len(spans)
    sp = np.ascontiguousarray(np.array([[a, b] for a, b, _ in spans] or [[0, 0]], dtype=np.int64))
    ro = np.ascontiguousarray(np.array([int(r) for _, _, r in spans] or [0], dtype=np.uint8))
    out = np.empty(max(L, 1), dtype=np.uint8)
    lib().or_span_members(L, P, n, _ptr(sp, P_I64), _ptr(ro, P_U8), _ptr(out, P_U8))
    return out[:L]
