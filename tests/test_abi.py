"""C-ABI boundary tests that need no GPU: the library loads, exports every
symbol include/sa.h declares, sizes workspaces on the host, and rejects bad
arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from sparse_attention_aware_b200 import _lib as L
from sparse_attention_aware_b200 import build as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "sa.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"SA_API\s+[\w\s\*]+?\b(sa_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L.EXPORTS)
    out = os.popen("nm -D --defined-only %s" % L.LIB_PATH).read()
    exported = set(re.findall(r" T (sa_\w+)", out))
    assert exported == set(names)


def test_status_strings(lib):
    for code in range(8):
        s = lib.sa_status_string(code).decode()
        assert s.startswith(L.STATUS_NAMES[code])
    assert lib.sa_version() >= 100


def _kv(batch=2, Hkv=2, d=128, P=16, max_pages=8, num_pages=16):
    # fake, aligned, never-dereferenced device addresses (host-side checks only)
    return L.KVCacheS(0x10000, 0x20000, 0x30000, 0x40000, batch, Hkv, d, P, max_pages, num_pages)


def _ws_bytes(lib, op, kv, **kw):
    q = L.WsQueryS(kw.get("num_q_heads", 0), kw.get("k", 0), kw.get("num_splits", 0),
                   kw.get("num_tokens", 0), kw.get("block_args", None))
    return lib.sa_workspace_bytes(op, ctypes.byref(kv), ctypes.byref(q))


def test_workspace_sizes(lib):
    kv = _kv()
    n = _ws_bytes(lib, L.OP_SELECT_TOPK, kv, num_q_heads=8, k=16)
    assert n == 256 + 2 * 8 * 8 * 16 * 4
    n = _ws_bytes(lib, L.OP_DECODE, kv, num_q_heads=8, num_splits=4)
    assert n % 256 == 0 and n >= 256 + 2 * 8 * 4 * 128 * 4 + 2 * 8 * 4 * 8
    assert _ws_bytes(lib, L.OP_DECODE, kv, num_q_heads=8, num_splits=65) == 0
    assert _ws_bytes(lib, L.OP_SELECT_TOPK, kv, num_q_heads=0, k=16) == 0
    bad = _kv(d=96)
    assert _ws_bytes(lib, L.OP_DECODE, bad, num_q_heads=8, num_splits=1) == 0
    a = L.BlockSelectArgsS()
    a.mode = L.SEL_RBS
    a.num_q_heads, a.num_tokens, a.block_size = 8, 1000, 64
    n_quant = _ws_bytes(lib, L.OP_SELECT_BLOCKS, _kv(P=64), block_args=ctypes.pointer(a))
    a.tau_c = a.tau_r = 0x50000
    n_expl = _ws_bytes(lib, L.OP_SELECT_BLOCKS, _kv(P=64), block_args=ctypes.pointer(a))
    assert n_quant > n_expl > 256


def _decode(lib, kv, Hq=8, splits=1, ws=0x100000, ws_bytes=1 << 30, sel=None, out=0x60000, q=0x70000,
            scale=0.1):
    if sel is None:
        sel = L.SelectionS(L.SEL_TOKENS, 0x80000, 0x90000, 16, None, None, 0)
    return lib.sa_sparse_decode_attn(ctypes.byref(kv), q, L.DTYPE_BF16, Hq, ctypes.byref(sel), scale,
                                     splits, out, None, ws, ws_bytes, None)


def test_host_validation_rejects_before_launch(lib):
    kv = _kv()
    INV, UNS, WS = 1, 2, 3
    assert _decode(lib, _kv(d=96)) == UNS
    assert _decode(lib, _kv(P=32)) == UNS
    assert _decode(lib, kv, Hq=3) == UNS                 # Hq % Hkv
    assert _decode(lib, kv, splits=0) == INV
    assert _decode(lib, kv, splits=65) == INV
    assert _decode(lib, kv, q=0x70001) == INV            # misaligned
    assert _decode(lib, kv, q=None) == INV
    assert _decode(lib, kv, scale=float("nan")) == INV
    assert _decode(lib, kv, ws=None) == WS
    assert _decode(lib, kv, ws=0x100010) == WS           # misaligned workspace
    assert _decode(lib, kv, ws_bytes=100) == WS
    bad_sel = L.SelectionS(7, 0x80000, 0x90000, 16, None, None, 0)
    assert _decode(lib, kv, sel=bad_sel) == INV
    kvbad = _kv()
    kvbad.k = None
    assert _decode(lib, kvbad) == INV
    # top-k
    r = lib.sa_select_topk(ctypes.byref(kv), 0x70000, L.DTYPE_BF16, 8, 0, 0x80000, 0x90000, 0x100000,
                           1 << 30, None)
    assert r == INV
    r = lib.sa_select_topk(ctypes.byref(kv), 0x70000, L.DTYPE_BF16, 32, 8, 0x80000, 0x90000, 0x100000,
                           1 << 30, None)
    assert r == UNS                                      # 16 q heads per kv head not built
    r = lib.sa_select_topk(ctypes.byref(kv), 0x70000, L.DTYPE_BF16, 8, 8, 0x80000, 0x90000, 0x100000,
                           64, None)
    assert r == WS
    # prefill
    kv64 = _kv(P=64)
    csr = L.BlockListS()
    csr.row_ptr, csr.cols, csr.nnz_capacity = 0x80000, 0x90000, 100
    pre = lambda kvx, T, causal, c=csr: lib.sa_sparse_prefill_attn(
        ctypes.byref(kvx), 0x70000, 8, T, ctypes.byref(c) if c is not None else None, 0.1, causal, 0x60000,
        None, 0x100000, 1 << 30, None)
    assert pre(kv, 100, 1) == UNS                        # prefill needs 64-token pages
    assert pre(kv64, 100, 0) == UNS                      # non-causal not built
    assert pre(kv64, 10_000, 1) == INV                   # more tokens than the cache holds
    assert pre(kv64, 100, 1, None) == INV                # no CSR
    bad = L.BlockListS()
    bad.row_ptr, bad.cols, bad.nnz_capacity = 0x80000, 0x90000, -1
    assert pre(kv64, 100, 1, bad) == INV
    # select_blocks
    a = L.BlockSelectArgsS()
    a.mode = 9
    o = L.BlockListS()
    assert lib.sa_select_blocks(ctypes.byref(kv), ctypes.byref(a), ctypes.byref(o), 0x100000, 1 << 30,
                                None) == INV
    a.mode = L.SEL_RBS
    a.num_q_heads, a.num_tokens, a.block_size, a.q = 8, 100, 32, 0x70000
    assert lib.sa_select_blocks(ctypes.byref(kv64), ctypes.byref(a), ctypes.byref(o), 0x100000, 1 << 30,
                                None) == UNS             # block size 32 not built
    a.block_size = 64
    a.p_c, a.p_r = 1.5, 0.9
    o.row_ptr, o.cols, o.nnz_capacity = 0x80000, 0x90000, 100
    assert lib.sa_select_blocks(ctypes.byref(kv64), ctypes.byref(a), ctypes.byref(o), 0x100000, 1 << 30,
                                None) == INV             # quantile outside [0, 1]
    a.p_c = 0.9
    for bad_scale in (0.0, -0.1, float("inf"), float("nan")):
        a.scale = bad_scale
        assert lib.sa_select_blocks(ctypes.byref(kv64), ctypes.byref(a), ctypes.byref(o), 0x100000, 1 << 30,
                                    None) == INV         # the selection scale must be finite and > 0
    a.mode = L.SEL_SPANS
    a.max_spans = 2000
    assert lib.sa_select_blocks(ctypes.byref(kv), ctypes.byref(a), ctypes.byref(o), 0x100000, 1 << 30,
                                None) == INV
    assert lib.sa_workspace_init(None, 256, None) == WS
    assert lib.sa_read_device_status(0x100010, None, None) == WS


def test_binding_fails_loudly_without_library(tmp_path):
    import importlib
    saved = L._lib
    try:
        L._lib = None
        with pytest.raises(ImportError):
            L.load(str(tmp_path / "missing.so"))
    finally:
        L._lib = saved


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "sa.h"

int main(void)
{
    if (sa_version() < 100) return 1;
    if (strncmp(sa_status_string(SA_OK), "SA_OK", 5) != 0) return 2;
    if (strncmp(sa_status_string(SA_ERR_WORKSPACE), "SA_ERR_WORKSPACE", 16) != 0) return 3;
    sa_kv_cache kv;
    memset(&kv, 0, sizeof kv);
    kv.k = (const void *)0x10000;
    kv.v = (const void *)0x20000;
    kv.page_table = (const int32_t *)0x30000;
    kv.seq_lens = (const int32_t *)0x40000;
    kv.batch = 2;
    kv.num_kv_heads = 2;
    kv.head_dim = 128;
    kv.page_size = 16;
    kv.max_pages_per_seq = 8;
    kv.num_pages = 16;
    sa_ws_query q;
    memset(&q, 0, sizeof q);
    q.num_q_heads = 8;
    q.k = 16;
    if (sa_workspace_bytes(SA_OP_SELECT_TOPK, &kv, &q) != 256 + 2 * 8 * 8 * 16 * 4) return 4;
    kv.head_dim = 96;
    if (sa_workspace_bytes(SA_OP_SELECT_TOPK, &kv, &q) != 0) return 5;
    puts("ok");
    return 0;
}
"""


def test_header_is_plain_c_and_links(lib, tmp_path):
    """include/sa.h compiles as C99 with no CUDA header, and a C program links
    libsa.so and calls its host-only entry points."""
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(L.LIB_PATH)
    inc = os.path.dirname(HEADER)
    import subprocess
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", inc, str(src), "-o", str(exe),
                    "-L", libdir, "-l:libsa.so", "-Wl,-rpath," + libdir], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


def test_binding_stream_wrapper_passes_calls_through():
    """Without ``stream=`` an entry point runs exactly as written; the wrapper
    keeps names and docstrings (it only enters the given stream's context)."""
    from sparse_attention_aware_b200 import api

    @api._on_call_stream
    def f(a, b=2, stream=None):
        """doc"""
        return a, b, stream

    assert f(1) == (1, 2, None) and f(1, b=3, stream=None) == (1, 3, None)
    assert f.__name__ == "f" and f.__doc__ == "doc"
    for name in ("select_topk", "sparse_decode_attn", "select_blocks_spans", "select_blocks_rbs",
                 "sparse_prefill_attn", "fetch_pages"):
        fn = getattr(api, name)
        assert fn.__name__ == name and fn.__wrapped__ is not None
