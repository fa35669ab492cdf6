"""Host-side checks of the C ABI: the library builds, loads and exports every
entry point of include/qsa.h, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    import torch  # noqa: F401  (loads the CUDA runtime the library links against)
    from top_sparse_attention_score_b200 import build, qsa
    build.build()
    return qsa.load()


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(qsa_\w+)\s*\(", src, flags=re.M)
    return names


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ["qsa_workspace_bytes", "qsa_cache_write", "qsa_decode", "qsa_prefill_chunk",
              "qsa_index_score", "qsa_topk_workspace_bytes", "qsa_topk", "qsa_attn", "qsa_merge",
              "qsa_last_error", "qsa_launch_count"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    from top_sparse_attention_score_b200 import qsa
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in qsa.SIGNATURES, f"binding lacks a signature for {name}"


def _fake_cache(qsa, cells=1000):
    # Aligned, non-NULL host addresses: only used by calls that must fail validation.
    return qsa.CacheStruct(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, cells)


def test_workspace_bytes(lib):
    assert lib.qsa_workspace_bytes(0, 0, 100, 10, 0) == 0
    assert lib.qsa_workspace_bytes(0, 9, 100, 10, 0) == 0          # n > 8
    assert lib.qsa_workspace_bytes(0, 1, 100, 0, 0) == 0           # top_k < 1
    assert lib.qsa_workspace_bytes(0, 1, 100, 10, 65) == 0         # nsplit > 64
    assert lib.qsa_workspace_bytes(2, 1, 100, 10, 0) == 0          # bad mode
    a = lib.qsa_workspace_bytes(0, 1, 4096, 512, 1)
    b = lib.qsa_workspace_bytes(0, 1, 65536, 512, 1)
    c = lib.qsa_workspace_bytes(0, 1, 65536, 512, 64)
    assert 0 < a < b < c
    # a decode step holds its rows' scores (rows * L * 4 bytes); a prompt chunk of more than
    # 8 rows holds candidate lists instead, well under its T x L score matrix
    assert lib.qsa_workspace_bytes(0, 8, 262144, 2048, 0) >= 8 * 262144 * 4
    pre = lib.qsa_workspace_bytes(1, 1024, 262144, 2048, 0)
    assert 0 < pre < 1024 * 262144 * 4 // 2
    assert lib.qsa_topk_workspace_bytes(4, 1000, 100) > 4 * 2048 * 4


def test_decode_rejects_bad_arguments(lib):
    from top_sparse_attention_score_b200 import qsa
    cs = _fake_cache(qsa)
    P = ctypes.c_void_p(0x60000)
    def call(L=1000, n=1, top_k=64, nsplit=0, ws_bytes=1 << 40, q=P, cache=ctypes.byref(cs), append=None,
             gate=None):
        return lib.qsa_decode(cache, L, n, append, q, P, P, gate, top_k, nsplit, 0.0625, P, ws_bytes, P, None,
                              None)
    assert call(n=0) == 1 and "n = 0" in qsa.last_error()
    assert call(n=9) == 1
    assert call(L=1001) == 1                      # beyond max_cells
    assert call(L=2, n=3) == 1                    # L < n
    assert call(top_k=0) == 1
    assert call(top_k=16385) == 1
    assert call(nsplit=65) == 1
    assert call(q=None) == 1
    assert call(q=ctypes.c_void_p(0x60004)) == 1  # misaligned
    assert call(ws_bytes=100) == 2 and "workspace" in qsa.last_error()
    assert call(cache=None) == 1
    bad = qsa.CacheStruct(0x10000, 0, 0x30000, 0x40000, 0x50000, 1000)
    assert call(cache=ctypes.byref(bad)) == 1
    half = qsa.NewCellsStruct(0x70000, 0, 0x80000)                # append with a NULL array
    assert call(append=ctypes.byref(half)) == 1 and "append" in qsa.last_error()
    assert call(gate=ctypes.c_void_p(0x60008)) == 1               # misaligned gate


def test_prefill_and_steps_reject_bad_arguments(lib):
    from top_sparse_attention_score_b200 import qsa
    cs = _fake_cache(qsa)
    P = ctypes.c_void_p(0x60000)
    cb = ctypes.byref(cs)
    def prefill(pos0, T, ws_bytes=1 << 40, cache=cb):
        return lib.qsa_prefill_chunk(cache, pos0, T, None, P, P, P, None, 64, 0.0625, P, ws_bytes, P, None, None)
    assert prefill(990, 20) == 1
    assert prefill(-1, 20) == 1
    assert prefill(0, 20, ws_bytes=10) == 2
    big = qsa.CacheStruct(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 1 << 20)
    assert prefill(0, 65536, cache=ctypes.byref(big)) == 1 and "65535" in qsa.last_error()  # grid limit
    assert lib.qsa_cache_write(cb, 999, 2, P, P, P, None) == 1
    assert lib.qsa_cache_write(cb, 0, 0, P, P, P, None) == 1
    assert lib.qsa_index_score(cb, 1, 100, P, P, P, 99, None) == 1       # ld < ncells
    assert lib.qsa_index_score(cb, 1, 100, P, P, P, 102, None) == 1      # ld % 4
    assert lib.qsa_index_score(cb, 1, 1001, P, P, P, 1004, None) == 1    # ncells > max_cells
    assert lib.qsa_topk(P, 100, 2, 100, 10, P, 1 << 40, P, None) == 1    # row 1 sees 101 > ld
    assert lib.qsa_topk(P, 100, 1, 0, 10, P, 1 << 40, P, None) == 1      # vis0 < 1
    assert lib.qsa_topk(P, 100, 1, 50, 10, P, 10, P, None) == 2
    assert lib.qsa_topk(P, 1 << 20, 65536, 50, 10, P, 1 << 40, P, None) == 1  # rows above 65535
    assert lib.qsa_attn(cb, 1, P, P, 64, 0, 0.0625, None, P, P, None) == 1
    assert lib.qsa_attn(cb, 1, P, P, 64, 2, 0.0625, None, None, P, None) == 1  # nsplit > 1 needs part
    assert lib.qsa_attn(cb, 1, P, P, 64, 1, 0.0625, None, P, None, None) == 1  # nsplit 1 needs out
    assert lib.qsa_attn(cb, 65536, P, P, 64, 1, 0.0625, None, P, P, None) == 1  # rows above 65535
    assert lib.qsa_merge(None, 1, 2, None, P, None) == 1
    assert lib.qsa_merge(P, 1, 65, None, P, None) == 1


def test_bench_split_rule_matches_the_library(lib):
    """bench.py reports the split count the library picks for nsplit = 0; the
    workspace holds the split partials, so its size shows which count was used."""
    import bench
    for n in range(1, 9):
        for k in (512, 2048):
            auto = lib.qsa_workspace_bytes(0, n, 65536, k, 0)
            assert auto == lib.qsa_workspace_bytes(0, n, 65536, k, bench.auto_nsplit(n, k)), (n, k)
            other = bench.auto_nsplit(n, k) + 1
            if other <= 64:
                assert auto != lib.qsa_workspace_bytes(0, n, 65536, k, other), (n, k)


def test_traffic_hash_follows_code_not_comments(tmp_path, monkeypatch):
    """A recorded DRAM-traffic figure stays valid through comment edits of its kernel's
    source and is dropped by any change to the code."""
    import bench
    csrc = tmp_path / "top_sparse_attention_score_b200" / "csrc"
    csrc.mkdir(parents=True)
    src = csrc / bench.KERNEL_SOURCES["merge_kernel"]
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = "// header\n#pragma once\n/* block\n comment */\nint f(int x) {  // trailing\n  return x + 1;\n}\n"
    src.write_text(base)
    h0 = bench.source_hash("merge_kernel")
    src.write_text(base.replace("// trailing", "// reworded").replace("block\n comment", "other text") + "\n\n")
    assert bench.source_hash("merge_kernel") == h0
    src.write_text(base.replace("x + 1", "x + 2"))
    assert bench.source_hash("merge_kernel") != h0


def test_static_topk_status_and_trace_reject_bad_arguments(lib):
    """The fixed-scratch selection's limits, the status read and the trace calls fail
    with QSA_ERR_ARG before any CUDA call."""
    from top_sparse_attention_score_b200 import qsa
    P = ctypes.c_void_p(0x60000)
    def static(ld=1024, rows=4, vis0=1000, top_k=64, scores=P, ids=P):
        return lib.qsa_topk_static(scores, ld, rows, vis0, top_k, ids, None)
    assert static(scores=None) == 1
    assert static(ids=None) == 1
    assert static(rows=0) == 1
    assert static(rows=9) == 1 and "fixed scratch" in qsa.last_error()   # above QSA_STATIC_MAX_ROWS
    assert static(top_k=0) == 1
    assert static(top_k=2049) == 1 and "fixed scratch" in qsa.last_error()  # above QSA_STATIC_MAX_TOPK
    assert static(vis0=0) == 1
    assert static(vis0=1022) == 1                                 # row 3 sees 1025 > ld
    assert static(ld=1026, vis0=100) == 1                         # ld % 4
    assert static(ids=ctypes.c_void_p(0x60004)) == 1              # misaligned
    assert lib.qsa_device_status(None, None) == 1
    assert lib.qsa_trace_begin(0, None) == 1
    assert lib.qsa_trace_begin(4097, None) == 1
    n = ctypes.c_int(-1)
    assert lib.qsa_trace_end(1, ctypes.byref(n), None, None) == 1 and "no trace" in qsa.last_error()


def test_cache_and_chunk_limits(lib):
    """A cache descriptor with misaligned arrays or an out-of-range size, and a prompt
    chunk's top_k outside [1, QSA_MAX_TOPK], are rejected before any launch."""
    from top_sparse_attention_score_b200 import qsa
    P = ctypes.c_void_p(0x60000)
    for cs in (qsa.CacheStruct(0x10008, 0x20000, 0x30000, 0x40000, 0x50000, 1000),  # misaligned k
               qsa.CacheStruct(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0),     # no cells
               qsa.CacheStruct(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, (1 << 24) + 1)):
        assert lib.qsa_cache_write(ctypes.byref(cs), 0, 1, P, P, P, None) == 1
        assert "cache" in qsa.last_error()
    cb = ctypes.byref(_fake_cache(qsa))
    for top_k in (0, 16385):
        assert lib.qsa_prefill_chunk(cb, 0, 20, None, P, P, P, None, top_k, 0.0625, P, 1 << 40, P,
                                     None, None) == 1
        assert "top_k" in qsa.last_error()
