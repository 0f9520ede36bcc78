"""Seeded synthetic workloads for head-aware sparse attention.

This module only draws random numbers and lays them out in the paged KV-cache
format; it contains none of the selection or attention arithmetic.  Both the
CUDA path (tests, bench) and the CPU oracle (tests, CPU baseline) consume the
tensors it produces, so it is the one piece the two sides share.

Every random stream is derived from ``(seed, stream id, sub id)`` through a
splitmix64 hash, so a given workload is reproducible on one device type.  The
CPU generator and the CUDA generator of torch produce different values for the
same seed; a test always builds its inputs on one device and hands the same
tensors to both sides.

Layouts (shared with the C ABI):
  * K, V cache : bf16 ``[num_pages][Hkv][P][d]`` -- one (page, kv head) tile is
    contiguous (``P*d*2`` bytes).
  * page table : int32 ``[B][max_pages_per_seq]`` (logical page -> physical page)
  * seq lens   : int32 ``[B]``
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import torch

from .cache import PagedCache  # noqa: F401  (re-exported: generators build caches)

# stream ids
S_Q, S_K, S_V, S_STRUCT, S_PERM, S_MODES, S_REDRAW, S_OUTLIER, S_PAD = range(1, 10)

_MASK64 = (1 << 64) - 1


def _splitmix64(x: int) -> int:
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def derive_seed(seed: int, stream: int, sub: int = 0) -> int:
    """63-bit seed for stream ``stream`` / sub-stream ``sub`` of ``seed``."""
    h = _splitmix64(seed & _MASK64)
    h = _splitmix64(h ^ (stream & _MASK64))
    h = _splitmix64(h ^ (sub & _MASK64))
    return h & ((1 << 63) - 1)


def generator(seed: int, stream: int, sub: int = 0, device="cpu") -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(derive_seed(seed, stream, sub))
    return g


def randn(shape, seed, stream, sub=0, device="cpu", dtype=torch.float32):
    g = generator(seed, stream, sub, device)
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(dtype)


# --------------------------------------------------------------------------
# paged cache
# --------------------------------------------------------------------------
def page_permutation(num_pages: int, seed: int, shuffle: bool, device="cpu") -> torch.Tensor:
    if not shuffle:
        return torch.arange(num_pages, dtype=torch.int64, device=device)
    g = generator(seed, S_PERM, 0, device)
    return torch.randperm(num_pages, generator=g, device=device)


def to_pages(logical: torch.Tensor, page_size: int, perm: torch.Tensor,
             extra_pages: int = 0, fill_seed: Optional[int] = None) -> torch.Tensor:
    """Scatter logical ``[B][Hkv][Lpad][d]`` rows into the paged pool.

    ``Lpad`` must be a multiple of ``page_size``.  Logical page ``p`` of sequence
    ``b`` goes to physical page ``perm[b*pps + p]``.  ``extra_pages`` unused
    pages are appended (filled from ``fill_seed``, or zeros).
    """
    B, H, Lp, d = logical.shape
    assert Lp % page_size == 0
    pps = Lp // page_size
    pages = logical.reshape(B, H, pps, page_size, d).permute(0, 2, 1, 3, 4).reshape(B * pps, H, page_size, d)
    total = B * pps + extra_pages
    out = torch.empty((total, H, page_size, d), dtype=logical.dtype, device=logical.device)
    if extra_pages:
        if fill_seed is None:
            out.zero_()
        else:
            out[:] = randn(out.shape, fill_seed, S_PAD, 0, logical.device, logical.dtype)
    out[perm[: B * pps]] = pages
    return out


def page_table_from_perm(B: int, pps: int, perm: torch.Tensor) -> torch.Tensor:
    return perm[: B * pps].reshape(B, pps).to(torch.int32).contiguous()


def make_cache(k_log: torch.Tensor, v_log: torch.Tensor, seq_lens: Sequence[int], page_size: int,
               seed: int, shuffle: bool = True, extra_pages: int = 0) -> PagedCache:
    """Build a :class:`PagedCache` from logical bf16 K/V ``[B][Hkv][Lpad][d]``."""
    B, H, Lp, d = k_log.shape
    pps = Lp // page_size
    perm = page_permutation(B * pps + extra_pages, seed, shuffle, k_log.device)
    k = to_pages(k_log, page_size, perm, extra_pages, seed)
    v = to_pages(v_log, page_size, perm, extra_pages, seed + 1)
    pt = page_table_from_perm(B, pps, perm)
    sl = torch.tensor(list(seq_lens), dtype=torch.int32, device=k_log.device)
    return PagedCache(k, v, pt, sl)


def repage_v(cache: PagedCache, v_log: torch.Tensor) -> torch.Tensor:
    """Lay a new logical V ``[B][Hkv][Lpad][d]`` out under ``cache``'s page table."""
    B, H, Lp, d = v_log.shape
    P = cache.page_size
    pps = Lp // P
    pages = v_log.reshape(B, H, pps, P, d).permute(0, 2, 1, 3, 4).reshape(B * pps, H, P, d)
    out = torch.zeros_like(cache.v)
    out[cache.page_table[:, :pps].reshape(-1).long()] = pages
    return out


def _pad_len(L: int, P: int) -> int:
    return ((L + P - 1) // P) * P


# --------------------------------------------------------------------------
# generic random decode cache (tests: ragged lengths, odd sizes)
# --------------------------------------------------------------------------
def random_decode(seed: int, B: int, Hq: int, Hkv: int, d: int, seq_lens: Sequence[int], P: int,
                  shuffle: bool = True, extra_pages: int = 3, q_dtype=torch.bfloat16, device="cpu"):
    """K, V ~ N(0,1) bf16 in a shuffled paged pool, Q ~ N(0,1) ``[B][Hq][d]``."""
    Lmax = max(max(seq_lens), 1)
    Lp = _pad_len(Lmax, P)
    k_log = randn((B, Hkv, Lp, d), seed, S_K, 0, device, torch.bfloat16)
    v_log = randn((B, Hkv, Lp, d), seed, S_V, 0, device, torch.bfloat16)
    cache = make_cache(k_log, v_log, seq_lens, P, seed, shuffle, extra_pages)
    q = randn((B, Hq, d), seed, S_Q, 0, device, q_dtype)
    return cache, q


# --------------------------------------------------------------------------
# Tiny decode: B=1, MHA 4 heads, d=64, L=4096, fp32 Q/K/V, 16 planted keys per
# head scaled x4 along q, top-k 256, anchor + 2 reuse layers.
# --------------------------------------------------------------------------
@dataclasses.dataclass
class DecodeWorkload:
    cache: PagedCache            # anchor layer's cache (K shared by all layers)
    v_layers: List[torch.Tensor] # paged V for every layer (index 0 = anchor)
    q_layers: List[torch.Tensor] # Q [B][Hq][d] for every layer
    k: int                       # top-k
    num_splits: int
    planted: Optional[torch.Tensor] = None   # int64 [B][Hkv][16] planted positions

    @property
    def num_q_heads(self) -> int:
        return int(self.q_layers[0].shape[1])


def planted_key(q_row: torch.Tensor, d: int) -> torch.Tensor:
    """Planted key along ``q``: 4 x the typical key norm (sqrt d)."""
    qn = q_row.double()
    return (4.0 * math.sqrt(d) * qn / qn.norm()).float()


def tiny_decode(seed: int = 1001, device="cpu", L: int = 4096, k: int = 256, layers: int = 3,
                n_planted: int = 16, q_subseed: Optional[List[int]] = None) -> DecodeWorkload:
    B, H, d, P = 1, 4, 64, 16
    Lp = _pad_len(L, P)
    k_log = randn((B, H, Lp, d), seed, S_K, 0, device, torch.float32)
    q_layers = [randn((B, H, d), seed, S_Q, li, device, torch.float32) for li in range(layers)]
    if q_subseed is not None:   # per-head redraws of the anchor query
        for h, sub in enumerate(q_subseed):
            if sub:
                q_layers[0][0, h] = randn((d,), seed, S_REDRAW, (h << 16) | sub, device, torch.float32)
    g = generator(seed, S_STRUCT, 0, device)
    planted = torch.stack([torch.randperm(L, generator=g, device=device)[:n_planted] for _ in range(H)])
    for h in range(H):
        k_log[0, h, planted[h]] = planted_key(q_layers[0][0, h], d).to(device)
    v_logs = [randn((B, H, Lp, d), seed, S_V, li, device, torch.float32) for li in range(layers)]
    cache = make_cache(k_log.to(torch.bfloat16), v_logs[0].to(torch.bfloat16), [L], P, seed, shuffle=False)
    v_layers = [cache.v] + [repage_v(cache, vl.to(torch.bfloat16)) for vl in v_logs[1:]]
    return DecodeWorkload(cache, v_layers, q_layers, k, 1, planted.unsqueeze(0))


# --------------------------------------------------------------------------
# GQA decode: K = eps + U_g z (rank-8 structure per kv head), Q, V ~ N(0,1) bf16
# --------------------------------------------------------------------------
def lowrank_keys(seed: int, B: int, Hkv: int, Lp: int, d: int, rank: int = 8, device="cpu",
                 b0: int = 0) -> torch.Tensor:
    U = randn((Hkv, d, rank), seed, S_STRUCT, 0, device) / math.sqrt(rank)
    out = torch.empty((B, Hkv, Lp, d), dtype=torch.bfloat16, device=device)
    for b in range(B):  # one batch row at a time keeps fp32 temporaries small
        eps = randn((Hkv, Lp, d), seed, S_K, b0 + b, device)
        z = randn((Hkv, Lp, rank), seed, S_STRUCT, 1 + b0 + b, device)
        out[b] = (eps + torch.einsum("gdr,glr->gld", U, z)).to(torch.bfloat16)
    return out


def gqa_decode(seed: int = 1002, device="cpu", B: int = 8, Hq: int = 32, Hkv: int = 8, d: int = 128,
               L: int = 32768, P: int = 16, k: int = 2048, layers: int = 4, num_splits: int = 8,
               seq_lens: Optional[Sequence[int]] = None, q_redraw: Optional[dict] = None) -> DecodeWorkload:
    """``q_redraw`` maps ``(b, h) -> sub`` to redraw that head's anchor query."""
    seq_lens = list(seq_lens) if seq_lens is not None else [L] * B
    Lp = _pad_len(max(seq_lens), P)
    k_log = lowrank_keys(seed, B, Hkv, Lp, d, 8, device)
    v_log0 = randn((B, Hkv, Lp, d), seed, S_V, 0, device, torch.bfloat16)
    cache = make_cache(k_log, v_log0, seq_lens, P, seed, shuffle=True)
    del k_log, v_log0
    q_layers = [randn((B, Hq, d), seed, S_Q, li, device, torch.bfloat16) for li in range(layers)]
    if q_redraw:
        for (b, h), sub in q_redraw.items():
            q_layers[0][b, h] = randn((d,), seed, S_REDRAW, (b << 40) | (h << 20) | sub, device, torch.bfloat16)
    v_layers = [cache.v]
    for li in range(1, layers):
        v_layers.append(repage_v(cache, randn((B, Hkv, Lp, d), seed, S_V, li, device, torch.bfloat16)))
    return DecodeWorkload(cache, v_layers, q_layers, k, num_splits)


# --------------------------------------------------------------------------
# Long-context masked decode (DA focus / local, LoZA streaming)
# --------------------------------------------------------------------------
MODE_FOCUS, MODE_LOCAL, MODE_STREAM, MODE_GLOBAL = 0, 1, 2, 3
MODE_NAMES = {MODE_FOCUS: "focus", MODE_LOCAL: "local", MODE_STREAM: "streaming", MODE_GLOBAL: "global"}


@dataclasses.dataclass
class MaskedDecodeWorkload:
    cache: PagedCache
    q_steps: torch.Tensor       # [steps][B][Hq][d] bf16
    modes: torch.Tensor         # int32 [steps][B]
    focus_chunks: torch.Tensor  # int32 [steps][B][2] (valid where mode == focus)
    chunk: int
    origin: int
    num_splits: int


def draw_modes(seed: int, steps: int, B: int, L: int, chunk: int, origin: int,
               modes=(MODE_FOCUS, MODE_LOCAL, MODE_STREAM), n_focus: int = 2):
    """Per (step, sequence): a mode uniform over ``modes`` and ``n_focus``
    distinct chunks drawn uniformly among the chunks that meet ``[0, L)``."""
    g = generator(seed, S_MODES, 0, "cpu")
    mode_ids = torch.tensor(modes, dtype=torch.int32)
    pick = torch.randint(0, len(modes), (steps, B), generator=g)
    out_modes = mode_ids[pick]
    # chunk c covers [origin + c*chunk, origin + (c+1)*chunk); those meeting [0, L)
    c_lo = math.floor((0 - origin) / chunk)
    c_hi = math.floor((L - 1 - origin) / chunk)
    n_chunks = c_hi - c_lo + 1
    fc = torch.zeros((steps, B, n_focus), dtype=torch.int32)
    for s in range(steps):
        for b in range(B):
            fc[s, b] = torch.randperm(n_chunks, generator=g)[:n_focus].to(torch.int32) + c_lo
    return out_modes, fc


def masked_decode(seed: int = 1003, device="cpu", B: int = 4, Hq: int = 64, Hkv: int = 8, d: int = 128,
                  L: int = 131072, P: int = 16, chunk: int = 2048, steps: int = 64, origin: int = 0,
                  num_splits: int = 8, seq_lens: Optional[Sequence[int]] = None,
                  modes=(MODE_FOCUS, MODE_LOCAL, MODE_STREAM)) -> MaskedDecodeWorkload:
    seq_lens = list(seq_lens) if seq_lens is not None else [L] * B
    Lp = _pad_len(max(seq_lens), P)
    k_log = randn((B, Hkv, Lp, d), seed, S_K, 0, device, torch.bfloat16)
    v_log = randn((B, Hkv, Lp, d), seed, S_V, 0, device, torch.bfloat16)
    cache = make_cache(k_log, v_log, seq_lens, P, seed, shuffle=True)
    del k_log, v_log
    q = randn((steps, B, Hq, d), seed, S_Q, 0, device, torch.bfloat16)
    m, fc = draw_modes(seed, steps, B, min(seq_lens), chunk, origin, modes)
    return MaskedDecodeWorkload(cache, q, m.to(device), fc.to(device), chunk, origin, num_splits)


# --------------------------------------------------------------------------
# Block-sparse causal prefill: clustered keys with outliers (mean dilution)
# --------------------------------------------------------------------------
@dataclasses.dataclass
class PrefillWorkload:
    cache: PagedCache      # B = 1, P = block size
    q: torch.Tensor        # bf16 [T][Hq][d]
    T: int
    block: int


def segment_clusters(seed: int, T: int, n_clusters: int, mean_seg: float, device="cpu") -> torch.Tensor:
    """Cluster id per token: segments of geometric length (mean ``mean_seg``),
    each with a uniformly drawn cluster."""
    g = generator(seed, S_STRUCT, 7, "cpu")
    n_seg_guess = int(T / mean_seg * 1.5) + 16
    p = 1.0 / mean_seg
    while True:
        u = torch.rand(n_seg_guess, generator=g, dtype=torch.float64)
        lens = torch.floor(torch.log1p(-u) / math.log1p(-p)).to(torch.int64) + 1
        if int(lens.sum()) >= T:
            break
        n_seg_guess *= 2
    cl = torch.randint(0, n_clusters, (lens.numel(),), generator=g)
    ids = torch.repeat_interleave(cl, lens)[:T]
    return ids.to(device)


def clustered_prefill(seed: int = 1004, device="cpu", T: int = 32768, Hq: int = 32, Hkv: int = 4,
                      d: int = 128, block: int = 64, n_clusters: int = 256, sigma: float = 0.3,
                      outlier_frac: float = 0.005, outlier_scale: float = 6.0, mean_seg: float = 256.0,
                      own_prob: float = 0.5, shuffle: bool = True) -> PrefillWorkload:
    """Keys: ``mu_m + sigma*eps`` with ``m`` the token's segment cluster; a
    fraction ``outlier_frac`` of keys is ``outlier_scale`` x a regular draw from
    a uniformly chosen other cluster.  Queries of head ``h`` (kv head ``g``):
    ``mu_{m'} + sigma*eps`` with ``m'`` the segment cluster w.p. ``own_prob``,
    else uniform.  V ~ N(0,1).  Cluster centres ``mu ~ N(0, I_d)`` per kv head."""
    P = block
    Tp = _pad_len(T, P)
    group = Hq // Hkv
    mu = randn((Hkv, n_clusters, d), seed, S_STRUCT, 1, device)
    seg = segment_clusters(seed, Tp, n_clusters, mean_seg, device)
    gk = generator(seed, S_OUTLIER, 0, device)
    is_out = torch.rand(Tp, generator=gk, device=device) < outlier_frac
    other = (seg + 1 + torch.randint(0, n_clusters - 1, (Tp,), generator=gk, device=device)) % n_clusters
    k_log = torch.empty((1, Hkv, Tp, d), dtype=torch.bfloat16, device=device)
    for gi in range(Hkv):
        eps = randn((Tp, d), seed, S_K, gi, device)
        cid = torch.where(is_out, other, seg)
        kk = mu[gi, cid] + sigma * eps
        kk = torch.where(is_out[:, None], outlier_scale * kk, kk)
        k_log[0, gi] = kk.to(torch.bfloat16)
    v_log = randn((1, Hkv, Tp, d), seed, S_V, 0, device, torch.bfloat16)
    cache = make_cache(k_log, v_log, [T], P, seed, shuffle=shuffle)
    del k_log, v_log
    q = torch.empty((Tp, Hq, d), dtype=torch.bfloat16, device=device)
    gq = generator(seed, S_Q, 1, device)
    for h in range(Hq):
        gi = h // group
        own = torch.rand(Tp, generator=gq, device=device) < own_prob
        rnd = torch.randint(0, n_clusters, (Tp,), generator=gq, device=device)
        cid = torch.where(own, seg, rnd)
        eps = randn((Tp, d), seed, S_Q, 100 + h, device)
        q[:, h] = (mu[gi, cid] + sigma * eps).to(torch.bfloat16)
    return PrefillWorkload(cache, q[:T].contiguous(), T, block)


def random_prefill(seed: int, T: int, Hq: int, Hkv: int, d: int, block: int, device="cpu",
                   shuffle: bool = True) -> PrefillWorkload:
    """Q, K, V ~ N(0,1) bf16 (tests)."""
    P = block
    Tp = _pad_len(T, P)
    k_log = randn((1, Hkv, Tp, d), seed, S_K, 0, device, torch.bfloat16)
    v_log = randn((1, Hkv, Tp, d), seed, S_V, 0, device, torch.bfloat16)
    cache = make_cache(k_log, v_log, [T], P, seed, shuffle=shuffle, extra_pages=2)
    q = randn((T, Hq, d), seed, S_Q, 0, device, torch.bfloat16)
    return PrefillWorkload(cache, q, T, block)
