"""Pins for the oracle's span membership and masked decode (CPU).

Golden round-out values from the pages' focus example, closed-form token
counts per mode, page constancy of rounded spans, overlap merging, and the
global span equal to dense attention (torch fp64 SDPA).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import modes as M
from sparse_attention_aware_b200 import workloads as W
from tests.helpers import dense_kv, sdpa64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "da_focus_roundout.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        rows.append([int(x) for x in line.split()])
    return rows


def test_golden_focus_roundout():
    for a, b, P, ra, rb, extra in _golden():
        L = 131072
        mem = oracle.span_members(L, P, [(a, b, True)])
        nz = np.nonzero(mem)[0]
        assert nz[0] == ra and nz[-1] + 1 == rb and len(nz) == rb - ra
        assert len(nz) - (b - a) == extra
        assert extra <= 2 * (P - 1)      # "at most a few dozen tokens per edge"


@pytest.mark.parametrize("L,P", [(131072, 16), (1000, 16), (4100, 64), (77, 16)])
def test_mode_token_counts(L, P):
    cnt = lambda spans: int(oracle.span_members(L, P, spans).sum())
    assert cnt(M.mode_spans(M.GLOBAL, L)) == L
    lo = L - 512
    if lo >= 0:
        assert cnt(M.mode_spans(M.LOCAL, L)) == L - (lo // P) * P
    if L >= 1028:
        assert cnt(M.mode_spans(M.STREAM, L)) == 4 + 1024
    else:
        assert cnt(M.mode_spans(M.STREAM, L)) == L


@pytest.mark.parametrize("origin", [0, 5, 2047])
def test_focus_chunks_closed_form_and_page_constancy(origin):
    L, P, C = 20000, 16, 2048
    for chunks in [(0, 3), (1, 2), (-1, 9)]:
        spans = M.mode_spans(M.FOCUS, L, C, origin, chunks)
        mem = oracle.span_members(L, P, spans)
        exp = 0
        cover = np.zeros(L, dtype=bool)
        for c in chunks:
            a = max(0, ((origin + c * C) // P) * P)
            b = min(L, -((-(origin + (c + 1) * C)) // P) * P)
            cover[a:max(a, b)] = True
        assert int(mem.sum()) == int(cover.sum())
        pages = mem[: (L // P) * P].reshape(-1, P)
        assert np.all((pages.min(1) == pages.max(1)))


def test_overlapping_spans_count_once():
    L, P = 300, 16
    mem = oracle.span_members(L, P, [(10, 100, True), (50, 120, True), (115, 117, False)])
    assert int(mem.sum()) == 128 - 0
    mem2 = oracle.span_members(L, P, [(0, 128, False)])
    assert np.array_equal(mem, mem2)


def test_global_span_decode_is_dense_and_local_is_suffix():
    cache, q = W.random_decode(31, 2, 4, 2, 32, [600, 333], 16)
    B, Hq, d = q.shape
    scale = 1 / math.sqrt(d)
    for mode in (M.GLOBAL, M.LOCAL):
        member = np.zeros((B, cache.max_pages * 16), dtype=np.uint8)
        for b in range(B):
            L = int(cache.seq_lens[b])
            member[b, :L] = oracle.span_members(L, 16, M.mode_spans(mode, L))
        out, _ = oracle.decode_members(cache, q, member, scale)
        out = out.reshape(B, Hq, d)
        for b in range(B):
            L = int(cache.seq_lens[b])
            lo = 0 if mode == M.GLOBAL else max(0, ((L - 512) // 16) * 16)
            for h in range(Hq):
                K, V = dense_kv(cache, b, h // 2, L)
                ref = sdpa64(q[b, h].double()[None], K[lo:], V[lo:], scale)[0]
                np.testing.assert_allclose(out[b, h], ref.numpy(), rtol=0, atol=1e-12)
