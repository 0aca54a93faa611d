"""CPU-side checks of the C-ABI library: it loads, exports every declared entry
point, reports its version and status names, sizes workspaces, and rejects
bad arguments on the host before touching the GPU."""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import pytest

from sparse_attention_weight_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^[\w \*]+?\b(dsa_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_weight_b200 import build
    build.build()
    return B.lib()


def test_library_exports_every_declared_function(lib):
    names = _declared_functions()
    assert set(B.EXPORTS) <= set(names) and len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n


def test_binding_constants_match_the_header():
    """The binding's op codes, status codes, device flags and limits are the
    header's (the binding restates them for Python callers)."""
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    defs = {n: int(v) for n, v in re.findall(r"^#define (DSA_\w+) (\d+)u?\b", src, flags=re.M)}
    enum = {n: int(v) for n, v in re.findall(r"^\s*(DSA_(?:OK|ERR_\w+)) = (\d+)", src, flags=re.M)}
    ops = {"DSA_OP_INDEXER": B.OP_INDEXER, "DSA_OP_TOPK": B.OP_TOPK, "DSA_OP_SPARSE_MLA": B.OP_SPARSE_MLA,
           "DSA_OP_FORWARD": B.OP_FORWARD, "DSA_OP_PROJECT": B.OP_PROJECT,
           "DSA_OP_MLA_BACKWARD": B.OP_MLA_BACKWARD, "DSA_OP_FORWARD_HOST": B.OP_FORWARD_HOST}
    for name, value in ops.items():
        assert defs[name] == value, name
    assert {n: v for n, v in defs.items() if n.startswith("DSA_OP_")} == ops
    assert defs["DSA_DEV_BAD_QUERY"] == B.DEV_BAD_QUERY and defs["DSA_DEV_BAD_INDEX"] == B.DEV_BAD_INDEX
    assert defs["DSA_DEV_TIMEOUT"] == B.DEV_TIMEOUT
    assert defs["DSA_NOALLOC_MAX_Q"] == B.NOALLOC_MAX_Q
    assert {v: n for n, v in enum.items()} == B.STATUS_NAMES and enum["DSA_OK"] == B.DSA_OK


def test_version_and_status_strings(lib):
    assert lib.dsa_abi_version() == 2
    for code, name in B.STATUS_NAMES.items():
        assert lib.dsa_status_string(code).decode() == name


def _fake_batch(T=16, Bn=2, max_len=3000, kv_rows=6000):
    # fake, aligned device addresses: never dereferenced by the failing calls below
    return B.DsaBatch(Bn, T, max_len, 0, kv_rows, 0x10000, 0x20000, 0x30000, 0x40000)


def test_workspace_sizes(lib):
    b = _fake_batch()
    sz = lambda op, **kw: lib.dsa_workspace_size(op, ctypes.byref(b), kw.get("hi", 64), kw.get("h", 128),
                                                 kw.get("k", 2048), kw.get("ld", 0))
    assert sz(B.OP_TOPK) >= 256
    assert sz(B.OP_INDEXER) >= 256 + (6 * 16 + 2) * 4
    fwd = sz(B.OP_FORWARD)
    assert fwd >= 16 * 3000 * 4 + 16 * 2048 * 4
    assert sz(B.OP_FORWARD, h=7) == 0 and sz(9) == 0
    assert lib.dsa_workspace_size(0, None, 64, 128, 2048, 0) == 0


def test_host_argument_checks(lib):
    b = _fake_batch()
    ws = 0x50000
    p = 0x60000
    big = 1 << 40
    # null batch / workspace
    assert lib.dsa_topk(None, p, 3000, 2048, p, ws, big, None) == 1
    assert lib.dsa_topk(ctypes.byref(b), p, 3000, 2048, p, None, big, None) == 1
    # unsupported shapes
    for hi in (0, 2, 10, 66, 68):        # H_I must be a multiple of 4 in [4, 64]
        assert lib.dsa_indexer_scores(ctypes.byref(b), p, p, p, hi, p, 3000, ws, big, None) == 2
    assert lib.dsa_indexer_scores(ctypes.byref(b), p, p, p, 64, p, 2999, ws, big, None) == 2   # ld % 4
    assert lib.dsa_indexer_scores(ctypes.byref(b), p, p, p, 64, p, 2000, ws, big, None) == 2   # ld < max_kv_len
    assert lib.dsa_topk(ctypes.byref(b), p, 3000, 4096, p, ws, big, None) == 2
    assert lib.dsa_topk(ctypes.byref(b), p, 3000, 0, p, ws, big, None) == 2
    assert lib.dsa_sparse_mla(ctypes.byref(b), p, p, p, 2048, 12, 0.1, p, None, ws, big, None) == 2
    assert lib.dsa_sparse_mla(ctypes.byref(b), p + 2, p, p, 2048, 128, 0.1, p, None, ws, big, None) == 2  # alignment
    # workspace too small
    assert lib.dsa_forward(ctypes.byref(b), p, p, p, 64, p, p, 128, 2048, 0.1, p, None, ws, 1024, None) == 3
    # bad batch fields
    bad = B.DsaBatch(0, 16, 3000, 0, 6000, 1, 1, 1, 1)
    assert lib.dsa_topk(ctypes.byref(bad), p, 3000, 2048, p, ws, big, None) == 1
    nulls = B.DsaBatch(2, 16, 3000, 0, 6000, 0, 0, 0, 0)
    assert lib.dsa_topk(ctypes.byref(nulls), p, 3000, 2048, p, ws, big, None) == 1


def test_paged_layout_host_checks(lib):
    """Paged caches (the block-table layout of paged inference caches): the page
    size must be a multiple of 64 dividing the physical rows, the page table
    must be given and cover max_kv_len; kv_offset is then not needed."""
    ws, p, big = 0x50000, 0x60000, 1 << 40
    pt = 0x70000

    def paged(page_size, pps, table=pt, kv_rows=8192, max_len=3000):
        return B.DsaBatch(2, 16, max_len, 0, kv_rows, 0, 0x20000, 0x30000, 0x40000, page_size, pps, table)

    sz = lambda b: lib.dsa_workspace_size(B.OP_FORWARD, ctypes.byref(b), 64, 128, 2048, 0)
    assert sz(paged(64, 47)) > 0                      # 47 * 64 = 3008 >= 3000
    assert sz(paged(64, 46)) == 0                     # 2944 < max_kv_len
    assert sz(paged(64, 47, table=0)) == 0            # no page table
    assert sz(B.DsaBatch(2, 16, 3000, 0, 8192, 0, 0x20000, 0x30000, 0x40000, -64, 47, pt)) == 0
    # unsupported page sizes: not a multiple of 64, or not dividing the physical rows
    for ps, pps in ((32, 94), (96, 32)):
        b = paged(ps, pps)
        assert lib.dsa_indexer_scores(ctypes.byref(b), p, p, p, 64, p, 3000, ws, big, None) == 2
        assert lib.dsa_sparse_mla(ctypes.byref(b), p, p, p, 2048, 128, 0.1, p, None, ws, big, None) == 2
        assert lib.dsa_forward(ctypes.byref(b), p, p, p, 64, p, p, 128, 2048, 0.1, p, None, ws, big, None) == 2
    b = paged(128, 24, kv_rows=8000)                  # 8000 rows is not whole pages of 128
    assert lib.dsa_sparse_mla(ctypes.byref(b), p, p, p, 2048, 128, 0.1, p, None, ws, big, None) == 2
    # the top-k reads no cache rows: any valid paged batch is accepted on the host
    assert lib.dsa_topk(ctypes.byref(paged(32, 94)), p, 3000, 2048, p, ws, 0, None) == 3


def test_project_append_host_checks(lib):
    b = _fake_batch()
    ws, p, big = 0x50000, 0x60000, 1 << 40
    sz = lib.dsa_workspace_size(B.OP_PROJECT, ctypes.byref(b), 64, 128, 0, 0)
    n_all = 64 * 128 + 128 + 64 + 576 + 128 * 576
    assert sz >= 256 + 16 * n_all * 4                 # the fp32 projections of the 16 tokens
    assert lib.dsa_workspace_size(B.OP_PROJECT, ctypes.byref(b), 10, 128, 0, 0) == 0
    call = lambda **kw: lib.dsa_project_append(ctypes.byref(b), kw.get("h", p), p, kw.get("d", 7168),
                                               kw.get("hi", 64), kw.get("H", 128), kw.get("base", 10000.0),
                                               p, p, p, p, p, ws, kw.get("ws_bytes", big), None)
    assert call(h=0) == 1                             # null input
    assert call(d=0) == 1 and call(base=0.0) == 1
    assert call(hi=10) == 2 and call(H=12) == 2 and call(d=7170) == 2
    assert call(h=p + 4) == 2                         # alignment
    assert call(ws_bytes=1024) == 3


def test_histogram_fusion_host_checks(lib):
    """dsa_indexer_scores_hist needs groups of <= 4 tokens of >= 32 padded heads;
    dsa_topk_uses_hist follows the top-k's kernel choice."""
    ws, p, big = 0x50000, 0x60000, 1 << 40
    b = _fake_batch()                                   # 16 queries, max_q_per_seq 0 (taken as 16)
    call = lambda bb, hi, hist=p: lib.dsa_indexer_scores_hist(ctypes.byref(bb), p, p, p, hi, p, 3000, hist, ws,
                                                              big if hist else 0, None)
    assert call(b, 64, hist=0) == 1                     # no histogram buffer
    assert call(b, 16) == 2                             # 16 heads: below 32 padded heads
    assert call(b, 32) == 2                             # 32 heads, 16 queries per sequence: groups of 8
    b4 = B.DsaBatch(2, 16, 3000, 4, 6000, 0x10000, 0x20000, 0x30000, 0x40000)
    assert call(b4, 32, hist=p + 4) == 2                # alignment of the histogram
    assert lib.dsa_topk_hist(ctypes.byref(b), p, 3000, 0, 2048, p, ws, big, None) == 1
    long_few = B.DsaBatch(16, 16, 131072, 1, 16 * 131072, 0x10000, 0x20000, 0x30000, 0x40000)
    short_many = B.DsaBatch(1, 8192, 8192, 8192, 8192, 0x10000, 0x20000, 0x30000, 0x40000)
    assert lib.dsa_topk_uses_hist(ctypes.byref(long_few), 2048) == 1      # clustered rows
    assert lib.dsa_topk_uses_hist(ctypes.byref(short_many), 2048) == 0    # rows cached per CTA
    assert lib.dsa_topk_uses_hist(None, 2048) == 0


def test_forward_host_host_checks(lib):
    """dsa_forward_host: the workspace covers the largest query chunk (a short last
    chunk may take split-KV partials that a full-size one does not), and bad
    arguments are refused before any copy is queued."""
    ws, p, big = 0x50000, 0x60000, 1 << 40
    for T in (16, 700, 5000):
        b = _fake_batch(T=T)
        host = lib.dsa_workspace_size(B.OP_FORWARD_HOST, ctypes.byref(b), 64, 128, 2048, 0)
        fwd = lib.dsa_workspace_size(B.OP_FORWARD, ctypes.byref(b), 64, 128, 2048, 0)
        assert host > 0 and fwd > 0
        # chunks of max(256, ceil(T/8)) queries: at most one chunk's scores and indices
        chunk = max(256, -(-T // 16))
        assert host >= min(T, chunk) * (3000 * 4 + 2048 * 4)
        assert host <= fwd + 64 * 2 * 128 * 512 * 4 + (1 << 20)
    assert lib.dsa_workspace_size(B.OP_FORWARD_HOST, ctypes.byref(_fake_batch()), 64, 12, 2048, 0) == 0
    b = _fake_batch()
    streams = (ctypes.c_void_p * 3)(None, None, None)
    call = lambda **kw: lib.dsa_forward_host(
        ctypes.byref(b), kw.get("hq", p), p, p, p, p, p, p, p, p, p, kw.get("hi", 64), 128, 2048, 0.1, p, None,
        kw.get("hout", p), ws, kw.get("ws_bytes", big), kw.get("streams", streams))
    assert call(streams=None) == 1                      # no stream array
    assert call(hq=0) == 1 and call(hout=0) == 1         # null host buffers
    assert call(hi=10) == 2
    assert call(ws_bytes=1024) == 3


def test_read_device_status_rejects_null(lib):
    flags = ctypes.c_uint32()
    assert lib.dsa_read_device_status(None, ctypes.byref(flags), None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(B, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        B.lib()
