"""Python view of the float64 CPU oracle for the QSA sparse-attention step.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg may use this package; the library never does.  The
arithmetic lives in ``qsa_oracle.cpp`` (plain C++, float64 accumulation);
this file only marshals numpy arrays into it.

Functions and the steps they follow (all from "opus r20 track A: MTP map
mlock + qsa_attn / qsa_merge decode tweaks" unless noted):

* ``index_scores``  -- the indexer score of every visible cell (the indexer
  query of section 3; qsa_score_mm in "opus r15 track A ...", item 1).
* ``topk`` / ``topk_fullsort`` -- per-token selection, ties to the lower index
  (qsa_topk, "opus r15 track A ...", item 1; one qids row per token in
  "Round 5 Track C Report ...", section 1, Target 2).
* ``attn_row`` -- max-subtracted softmax attention over int8 K/V with fp16
  scales (qsa_attn, section 2; data types in section 3).
* ``partials_row`` / ``merge_row`` -- split partials and their log-sum-exp
  merge (qsa_merge, section 2).
* ``dense_attn_row`` -- brute-force softmax over every visible cell.
* ``gate_row`` -- the output gate, O * sigmoid(gate) ("attention + gate",
  section 3).
* ``quantize`` / ``cache_write`` -- the int8 + per-32 fp16 scale quantizer.
* ``rows`` -- the whole step for chosen rows of a call.

Parity status: every function is pinned by tests/test_oracle_pins.py
(closed forms, invariants, brute force, hand-worked fixtures in
tests/golden/).  The pages print no worked QSA values, so no pin comes
from them directly.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def configure(L):
    """Declare the argument types of an oracle library handle (ctypes.CDLL)."""
    P = ctypes.c_void_p
    i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
    L.qsa_oracle_half_to_double.restype = dbl
    L.qsa_oracle_half_to_double.argtypes = [ctypes.c_uint16]
    L.qsa_oracle_float_to_half.restype = ctypes.c_uint16
    L.qsa_oracle_float_to_half.argtypes = [ctypes.c_float]
    L.qsa_oracle_index_scores.argtypes = [P, i64, P, P, P]
    L.qsa_oracle_topk.argtypes = [P, i64, i32, P]
    L.qsa_oracle_topk.restype = i32
    L.qsa_oracle_topk_fullsort.argtypes = [P, i64, i32, P]
    L.qsa_oracle_topk_fullsort.restype = i32
    L.qsa_oracle_attn_row.argtypes = [P, P, P, P, P, P, i32, dbl, P]
    L.qsa_oracle_partials_row.argtypes = [P, P, P, P, P, P, i32, i32, dbl, P, P, P]
    L.qsa_oracle_merge_row.argtypes = [P, P, P, i32, P]
    L.qsa_oracle_dense_attn_row.argtypes = [P, P, P, P, i64, P, dbl, P]
    L.qsa_oracle_quantize.argtypes = [P, i64, P, P]
    L.qsa_oracle_cache_write.argtypes = [P, P, P, P, P, i64, i32, P, P, P]
    L.qsa_oracle_gate_row.argtypes = [P, P]
    L.qsa_oracle_rows.argtypes = [P, P, P, P, P, i64, P, i32, P, P, P, P, i32, dbl, P, P, P, i64, i32]
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(_build.build()))
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a).view(np.uint16)


def half_to_double(bits: np.ndarray) -> np.ndarray:
    L = lib()
    return np.array([L.qsa_oracle_half_to_double(int(b)) for b in np.asarray(bits).ravel()])


def float_to_half_bits(x: np.ndarray) -> np.ndarray:
    L = lib()
    return np.array([L.qsa_oracle_float_to_half(float(v)) for v in np.asarray(x, np.float32).ravel()],
                    dtype=np.uint16)


def index_scores(keys: np.ndarray, V: int, iq: np.ndarray, iw: np.ndarray) -> np.ndarray:
    keys = np.ascontiguousarray(keys, np.float16)
    iq = np.ascontiguousarray(iq, np.float16)
    iw = np.ascontiguousarray(iw, np.float32)
    out = np.empty(V, np.float64)
    lib().qsa_oracle_index_scores(_p(_u16(keys)), V, _p(_u16(iq)), _p(iw), _p(out))
    return out


def topk(scores: np.ndarray, k: int) -> np.ndarray:
    s = np.ascontiguousarray(scores, np.float64)
    ids = np.empty(k, np.int32)
    lib().qsa_oracle_topk(_p(s), s.size, k, _p(ids))
    return ids


def topk_fullsort(scores: np.ndarray, k: int) -> np.ndarray:
    s = np.ascontiguousarray(scores, np.float64)
    ids = np.empty(k, np.int32)
    lib().qsa_oracle_topk_fullsort(_p(s), s.size, k, _p(ids))
    return ids


def _cache_ptrs(cache):
    k = np.ascontiguousarray(cache.k)
    v = np.ascontiguousarray(cache.v)
    ks = _u16(np.ascontiguousarray(cache.ks, np.float16))
    vs = _u16(np.ascontiguousarray(cache.vs, np.float16))
    keep = (k, v, ks, vs)
    return keep, (_p(k), _p(v), _p(ks), _p(vs))


def attn_row(cache, q: np.ndarray, ids: np.ndarray, scale: float) -> np.ndarray:
    keep, ptrs = _cache_ptrs(cache)
    q = np.ascontiguousarray(q, np.float32)
    ids = np.ascontiguousarray(ids, np.int32)
    out = np.empty((24, 256), np.float64)
    lib().qsa_oracle_attn_row(*ptrs, _p(q), _p(ids), ids.size, scale, _p(out))
    return out


def partials_row(cache, q: np.ndarray, ids: np.ndarray, nsplit: int, scale: float):
    keep, ptrs = _cache_ptrs(cache)
    q = np.ascontiguousarray(q, np.float32)
    ids = np.ascontiguousarray(ids, np.int32)
    m = np.empty((24, nsplit), np.float64)
    l = np.empty((24, nsplit), np.float64)
    o = np.empty((24, nsplit, 256), np.float64)
    lib().qsa_oracle_partials_row(*ptrs, _p(q), _p(ids), ids.size, nsplit, scale, _p(m), _p(l), _p(o))
    return m, l, o


def merge_row(m: np.ndarray, l: np.ndarray, o: np.ndarray) -> np.ndarray:
    m = np.ascontiguousarray(m, np.float64)
    l = np.ascontiguousarray(l, np.float64)
    o = np.ascontiguousarray(o, np.float64)
    out = np.empty((24, 256), np.float64)
    lib().qsa_oracle_merge_row(_p(m), _p(l), _p(o), m.shape[1], _p(out))
    return out


def dense_attn_row(cache, V: int, q: np.ndarray, scale: float) -> np.ndarray:
    keep, ptrs = _cache_ptrs(cache)
    q = np.ascontiguousarray(q, np.float32)
    out = np.empty((24, 256), np.float64)
    lib().qsa_oracle_dense_attn_row(*ptrs, V, _p(q), scale, _p(out))
    return out


def gate_row(out: np.ndarray, gate: np.ndarray) -> np.ndarray:
    """out [24][256] times sigmoid(gate [24][256]) (a new array)."""
    res = np.array(out, np.float64, copy=True, order="C")
    g = np.ascontiguousarray(gate, np.float32)
    assert res.shape == (24, 256) and g.shape == (24, 256)
    lib().qsa_oracle_gate_row(_p(g), _p(res))
    return res


def quantize(x: np.ndarray):
    x = np.ascontiguousarray(x, np.float32).ravel()
    assert x.size % 32 == 0
    q = np.empty(x.size, np.int8)
    s = np.empty(x.size // 32, np.uint16)
    lib().qsa_oracle_quantize(_p(x), x.size // 32, _p(q), _p(s))
    return q, s


def cache_write(cache, pos0: int, k: np.ndarray, v: np.ndarray, key: np.ndarray) -> None:
    """Quantize and append n cells into ``cache`` (modified in place)."""
    k = np.ascontiguousarray(k, np.float32)
    v = np.ascontiguousarray(v, np.float32)
    key = _u16(np.ascontiguousarray(key, np.float16))
    n = k.shape[0]
    assert cache.ks.dtype == np.float16 and cache.ks.flags["C_CONTIGUOUS"]
    lib().qsa_oracle_cache_write(_p(cache.k), _p(cache.v), _p(cache.ks.view(np.uint16)),
                                 _p(cache.vs.view(np.uint16)), _p(cache.idx_key.view(np.uint16)),
                                 pos0, n, _p(k), _p(v), _p(key))


def rows(wl, row_ids=None, want_scores: bool = False, threads: int | None = None, top_k=None, gate=None):
    """Run the whole step for the given rows of workload ``wl`` (synth.Workload);
    ``gate`` (float32 [wl.rows][24][256]) gates the outputs.

    Returns (out [nr][24][256] float64, ids [nr][top_k] int32, scores or None).
    """
    if row_ids is None:
        row_ids = np.arange(wl.rows)
    row_ids = np.ascontiguousarray(row_ids, np.int32)
    k = wl.top_k if top_k is None else top_k
    nr = row_ids.size
    keep, ptrs = _cache_ptrs(wl.cache)
    key = _u16(np.ascontiguousarray(wl.cache.idx_key, np.float16))
    q = np.ascontiguousarray(wl.q, np.float32)
    iq = _u16(np.ascontiguousarray(wl.iq, np.float16))
    iw = np.ascontiguousarray(wl.iw, np.float32)
    out = np.empty((nr, 24, 256), np.float64)
    ids = np.empty((nr, k), np.int32)
    vis0 = wl.vis0()
    ld = vis0 + int(row_ids.max()) if nr else 0
    scores = np.empty((nr, ld), np.float64) if want_scores else None
    threads = threads or (os.cpu_count() or 1)
    g = None if gate is None else np.ascontiguousarray(gate, np.float32)
    lib().qsa_oracle_rows(*ptrs, _p(key), vis0, _p(row_ids), nr, _p(q), _p(iq), _p(iw),
                          None if g is None else _p(g), k, wl.scale,
                          _p(out), _p(ids), _p(scores) if scores is not None else None, ld, threads)
    return out, ids, scores
