"""Pins for the CPU oracle: checks against facts fixed outside the oracle itself.

Every check raises AssertionError on failure.  ``test_oracle_pins`` runs them
against the oracle; ``test_oracle_mutants`` runs them against copies of the
oracle with one planted mistake each and requires at least one to fail.

Sources of truth used (none of them re-types the oracle's own formula):
* hand-worked fixtures in tests/golden/ (derivations inline);
* the IEEE binary16 format as implemented independently by numpy;
* closed forms (one selected cell, identical keys, one-hot keys, zero scale);
* brute force on tiny inputs (all subsets for the selection rule);
* invariants: split count, causal mask, id order, padding.
"""
from __future__ import annotations

import itertools
import math
import os

import numpy as np

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- fp16 format

def check_half_decode_exhaustive():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = oracle.half_to_double(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zero kept
    assert math.copysign(1.0, got[0x8000]) == -1.0


def check_float_to_half_rn():
    st = synth.Stream(7, "f2h")
    x = np.concatenate([
        st.normal(3000) * 10.0 ** st.integers(3000, 12).astype(np.float64) / 1e6,
        np.array([65504.0, 65519.0, 65520.0, 1e9, -65520.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
                  2.0 ** -14, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, -0.0, 0.0]),
    ]).astype(np.float32)
    got = oracle.float_to_half_bits(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- quantizer

def _parse_sparse(tok: str, n: int) -> np.ndarray:
    out = np.zeros(n, np.float64)
    for t in tok.split():
        i, v = t.split(":")
        out[int(i)] = float(v)
    return out


def load_quantize_golden():
    cases = []
    with open(os.path.join(GOLDEN, "quantize_hand.txt")) as f:
        for line in f:
            if not line.startswith("group "):
                continue
            parts = [p.strip() for p in line.split("|")]
            name = parts[0].split()[1]
            x = _parse_sparse(parts[1], 32).astype(np.float32)
            sbits = int(parts[2].split()[1], 16)
            codes = _parse_sparse(parts[3][len("codes"):], 32).astype(np.int8)
            cases.append((name, x, sbits, codes))
    return cases


def check_quantize_golden():
    cases = load_quantize_golden()
    assert len(cases) >= 7
    for name, x, sbits, codes in cases:
        q, s = oracle.quantize(x)
        assert int(s[0]) == sbits, (name, hex(int(s[0])), hex(sbits))
        assert np.array_equal(q, codes), (name, q, codes)


def check_quantize_patterns():
    pats = synth.quantizer_patterns(11, 512)
    for name, x in pats.items():
        q, s = oracle.quantize(x)
        sc = s.view(np.float16).astype(np.float64)
        assert np.all(np.abs(q.astype(np.int32)) <= 127), name
        xg = x.reshape(-1, 32).astype(np.float64)
        qg = q.reshape(-1, 32).astype(np.float64)
        amax = np.abs(xg).max(1)
        zero = sc == 0
        assert np.all(qg[zero] == 0), name
        # round trip: every value within half a scale step of its code, plus whatever the
        # clamp at +-127 cuts off when the fp16 scale rounded below amax/127
        s2 = sc[:, None]
        err = np.abs(xg - qg * s2)
        excess = np.maximum(0.0, np.abs(xg) - 127.5 * s2)
        bound = 0.5 * s2 * (1 + 2.0 ** -20) + excess + np.abs(xg) * 2.0 ** -23
        assert np.all((err <= bound) | zero[:, None]), name
        # a group with a normal fp16 scale reaches +-127 exactly at its largest value
        normal = sc >= 2.0 ** -14
        assert np.all(np.abs(qg[normal]).max(1) == 127), name
        # the scale is the fp16 value nearest amax/127 (numpy's own fp16 rounding)
        ratio = (amax.astype(np.float32) / np.float32(127.0)).astype(np.float32)
        ref = np.minimum(ratio.astype(np.float16).astype(np.float64), 65504.0)
        assert np.array_equal(sc, ref), name
        # sign symmetry: quantizing -x negates every code and keeps the scale
        qn, sn = oracle.quantize(-x)
        assert np.array_equal(sn, s) and np.array_equal(qn, (-q.astype(np.int16)).astype(np.int8)), name


def check_cache_write_layout():
    cells, pos0, n = 16, 5, 3
    cache = synth.make_cache(21, cells)
    before = [a.copy() for a in (cache.k, cache.v, cache.ks, cache.vs, cache.idx_key)]
    k, v, key = synth.make_new_cells(22, n)
    oracle.cache_write(cache, pos0, k, v, key)
    after = (cache.k, cache.v, cache.ks, cache.vs, cache.idx_key)
    inside = np.zeros(cells, bool)
    inside[pos0:pos0 + n] = True
    for b, a in zip(before, after):
        assert np.array_equal(b[~inside], a[~inside])          # untouched outside the target cells
    assert np.array_equal(cache.idx_key[pos0:pos0 + n], key)
    for i in range(n):
        for g in range(2):
            qk, sk = oracle.quantize(k[i, g])
            qv, sv = oracle.quantize(v[i, g])
            assert np.array_equal(cache.k[pos0 + i, g], qk)
            assert np.array_equal(cache.v[pos0 + i, g], qv)
            assert np.array_equal(cache.ks[pos0 + i, g].view(np.uint16), sk)
            assert np.array_equal(cache.vs[pos0 + i, g].view(np.uint16), sv)
            # group j of 32 values owns scale j: a value scaled up in group 3 only moves scale 3
            bumped = k[i, g].copy()
            bumped[3 * 32:4 * 32] *= 4.0
            _, sb = oracle.quantize(bumped)
            changed = np.nonzero(sb != sk)[0]
            assert set(changed.tolist()) <= {3} and changed.size == 1


# ---------------------------------------------------------------- indexer score

def check_index_score_golden():
    iq = np.zeros((4, 64))
    keys = {}
    with open(os.path.join(GOLDEN, "index_score_hand.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            head, body = [p.strip() for p in line.split("|", 1)]
            if head.startswith("iq"):
                iq[int(head.split()[1])] = _parse_sparse(body, 64)
            elif head == "w":
                w = np.array([float(t) for t in body.split()])
            elif head.startswith("key"):
                keys[int(head.split()[1])] = _parse_sparse(body, 64)
            elif head == "expect":
                expect = np.array([float(t) for t in body.split()])
    K = np.stack([keys[i] for i in range(len(keys))]).astype(np.float16)
    got = oracle.index_scores(K, K.shape[0], iq.astype(np.float16), w.astype(np.float32))
    assert np.array_equal(got, expect), (got, expect)


def check_index_score_onehot():
    # key c = e_(c mod 64): the dot with head h is iq[h][c mod 64], so the score is
    # sum_h w_h * max(0, iq[h][c mod 64]) -- one column of iq at a time.
    st = synth.Stream(31, "onehot")
    iq = st.normal(256).reshape(4, 64).astype(np.float16)
    w = st.uniform(4).astype(np.float32)
    V = 130
    keys = np.zeros((V, 64), np.float16)
    keys[np.arange(V), np.arange(V) % 64] = 1.0
    got = oracle.index_scores(keys, V, iq, w)
    col = iq.astype(np.float64)[:, np.arange(V) % 64]                 # [4][V]
    expect = np.zeros(V)
    for h in range(4):
        expect += float(w[h]) * np.where(col[h] > 0, col[h], 0.0)
    assert np.allclose(got, expect, rtol=0, atol=1e-15)
    # only visible cells are read: a shorter V gives the prefix
    assert np.array_equal(oracle.index_scores(keys, 17, iq, w), got[:17])
    # positive homogeneity: doubling every weight doubles every score
    assert np.array_equal(oracle.index_scores(keys, V, iq, (2 * w).astype(np.float32)), 2 * got)


# ---------------------------------------------------------------- selection

def _is_topk(scores, ids, k):
    """The selection rule, checked by brute force over every (in, out) pair."""
    V = len(scores)
    take = min(k, V)
    sel = [i for i in ids if i >= 0]
    if len(sel) != take or sorted(sel) != list(sel) or len(set(sel)) != take:
        return False
    if any(i != -1 for i in ids[take:]):
        return False
    s = set(sel)
    for a in s:
        for b in range(V):
            if b in s:
                continue
            if not (scores[a] > scores[b] or (scores[a] == scores[b] and a < b)):
                return False
    return True


def check_topk_bruteforce():
    st = synth.Stream(41, "topk")
    for trial in range(60):
        V = 1 + int(st.integers(1, 12)[0])
        k = 1 + int(st.integers(1, 14)[0])
        scores = (st.integers(V, 4) - 1).astype(np.float64)            # many ties
        ids = oracle.topk(scores, k)
        assert _is_topk(list(scores), list(ids), k), (scores, k, ids)
        # exactly one subset satisfies the rule: enumerate them all
        take = min(k, V)
        good = [c for c in itertools.combinations(range(V), take)
                if _is_topk(list(scores), list(c) + [-1] * (k - take), k)]
        assert good == [tuple(int(i) for i in ids[:take])]
        assert np.array_equal(oracle.topk_fullsort(scores, k), ids)


def check_topk_special():
    # all equal -> the lowest indices
    assert np.array_equal(oracle.topk(np.zeros(10), 4), np.arange(4))
    # fewer visible than k -> all visible, padded with -1
    assert np.array_equal(oracle.topk(np.array([3.0, 1.0, 2.0]), 5), [0, 1, 2, -1, -1])
    # strictly decreasing -> the first k
    assert np.array_equal(oracle.topk(np.arange(20, 0, -1).astype(float), 6), np.arange(6))
    # increasing -> the last k, reported ascending
    assert np.array_equal(oracle.topk(np.arange(20).astype(float), 6), np.arange(14, 20))
    # signed zero ties with zero
    assert np.array_equal(oracle.topk(np.array([0.0, -0.0, 0.0, -1.0]), 2), [0, 1])
    # larger random case: both selectors agree
    st = synth.Stream(43, "topk2")
    s = np.round(st.normal(5000) * 4) / 4
    for k in (1, 7, 100, 2048, 4999, 5000, 6000):
        assert np.array_equal(oracle.topk(s, k), oracle.topk_fullsort(s, k))


# ---------------------------------------------------------------- attention

def _small_cache(seed, cells, **kw):
    return synth.make_cache(seed, cells, **kw)


def _deq(a, s):
    return a.astype(np.float64) * np.repeat(s.astype(np.float64), 32, axis=-1)


def check_attn_single_cell():
    # one selected cell: softmax weight 1, O[h] = its dequantised V row of KV head h // 12
    cache = _small_cache(51, 40)
    q, _, _ = synth.make_queries(52, 1)
    for c in (0, 17, 39):
        out = oracle.attn_row(cache, q[0], np.array([c, -1, -1], np.int32), 1 / 16)
        vd = _deq(cache.v[c], cache.vs[c])                             # [2][256]
        for h in range(24):
            assert np.array_equal(out[h], vd[h // 12]), (c, h)


def check_attn_uniform():
    # identical K rows and scales for every cell: all scores tie, O = mean of dequantised V
    cache = _small_cache(53, 30)
    cache.k[:] = cache.k[0]
    cache.ks[:] = cache.ks[0]
    q, _, _ = synth.make_queries(54, 1)
    ids = np.array([2, 5, 9, 11, 29], np.int32)
    out = oracle.attn_row(cache, q[0], ids, 1 / 16)
    vd = _deq(cache.v[ids], cache.vs[ids])                            # [5][2][256]
    for h in range(24):
        assert np.allclose(out[h], vd[:, h // 12].mean(0), rtol=1e-13, atol=1e-15)
    # scale 0 makes any K uniform too
    cache2 = _small_cache(55, 30)
    out0 = oracle.attn_row(cache2, q[0], ids, 0.0)
    vd2 = _deq(cache2.v[ids], cache2.vs[ids])
    for h in range(24):
        assert np.allclose(out0[h], vd2[:, h // 12].mean(0), rtol=1e-13, atol=1e-15)


def check_attn_dominant():
    # q along one cell's dequantised key, large: that cell takes (almost) all the weight
    cache = _small_cache(57, 64)
    kd = _deq(cache.k, cache.ks)                                       # [64][2][256]
    c = 23
    q = np.zeros((24, 256), np.float32)
    for h in range(24):
        q[h] = (kd[c, h // 12] / np.linalg.norm(kd[c, h // 12]) * 4000.0).astype(np.float32)
    out = oracle.attn_row(cache, q, np.arange(64, dtype=np.int32), 1 / 16)
    vd = _deq(cache.v[c], cache.vs[c])
    for h in range(24):
        assert np.allclose(out[h], vd[h // 12], rtol=0, atol=1e-6 * np.abs(vd).max())


def check_attn_gqa_and_groups():
    # V of KV head 1 constant 1 with scale 2 in group 3 only: heads 12..23 read 2 on d in [96, 128)
    cache = _small_cache(59, 8)
    cache.v[:, 1] = 1
    cache.vs[:, 1] = np.float16(1.0)
    cache.vs[:, 1, 3] = np.float16(2.0)
    q, _, _ = synth.make_queries(60, 1)
    out = oracle.attn_row(cache, q[0], np.arange(8, dtype=np.int32), 1 / 16)
    for h in range(12, 24):
        expect = np.ones(256)
        expect[96:128] = 2.0
        assert np.allclose(out[h], expect, rtol=1e-14)
    # heads 0..11 use KV head 0 and so differ from the constant
    assert not np.allclose(out[0], 1.0)
    # K scale group g multiplies d in [32g, 32g+32): zero q outside group 5 and zero ks[5] -> uniform
    cache2 = _small_cache(61, 8)
    cache2.ks[:, :, 5] = np.float16(0.0)
    q2 = np.zeros((24, 256), np.float32)
    q2[:, 160:192] = 50.0
    out2 = oracle.attn_row(cache2, q2, np.arange(8, dtype=np.int32), 1 / 16)
    vd = _deq(cache2.v, cache2.vs)
    for h in range(24):
        assert np.allclose(out2[h], vd[:, h // 12].mean(0), rtol=1e-13, atol=1e-15)


def check_attn_order_and_padding():
    cache = _small_cache(63, 50)
    q, _, _ = synth.make_queries(64, 1)
    ids = np.array([3, 8, 10, 21, 33, 47], np.int32)
    base = oracle.attn_row(cache, q[0], ids, 1 / 16)
    perm = ids[[4, 0, 5, 2, 1, 3]]
    assert np.allclose(oracle.attn_row(cache, q[0], perm, 1 / 16), base, rtol=1e-13, atol=1e-16)
    padded = np.concatenate([ids, -np.ones(5, np.int32)])
    assert np.array_equal(oracle.attn_row(cache, q[0], padded, 1 / 16), base)


def load_softmax_golden():
    """The hand-worked softmax fixture: per-KV-head weights and V codes, the expected
    outputs and the two-piece partials (tests/golden/attn_softmax_hand.txt)."""
    vals, pieces = {}, {}
    with open(os.path.join(GOLDEN, "attn_softmax_hand.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            head, body = [p.strip() for p in line.split("|", 1)]
            if head.startswith("piece"):
                g = int(head.split()[1][1:])
                fields = [p.split() for p in line.split("|")[1:]]
                pieces[g] = {f[0]: np.array([float(t) for t in f[1:]]) for f in fields}
            else:
                vals[head] = np.array([float(t) for t in body.split()])
    return vals, pieces


def softmax_golden_case():
    """Cache, query and ids of the hand-worked softmax fixture (construction in the file)."""
    vals, pieces = load_softmax_golden()
    cache = synth.make_cache(81, 4)
    cache.k[:] = 0
    for c in range(4):
        cache.k[c, :, c] = 1
    cache.ks[:] = np.float16(1.0)
    for g in range(2):
        cache.v[:, g, :] = vals[f"a{g}"].astype(np.int8)[:, None]
    cache.vs[:] = (2.0 ** -np.arange(8)).astype(np.float16)
    q = np.zeros((24, 256), np.float32)
    for h in range(24):
        q[h, :4] = (16.0 * np.log(vals[f"w{h // 12}"])).astype(np.float32)
    return cache, q, vals, pieces


def check_attn_softmax_golden():
    # logits ln w_c give softmax weights w_c / sum(w): pins the natural exp, the 1/16 scale
    # applied to the dot product and the max subtraction, which the closed forms above
    # (one cell, uniform, dominant) cannot tell apart
    cache, q, vals, pieces = softmax_golden_case()
    ids = np.arange(4, dtype=np.int32)
    dims = 2.0 ** -(np.arange(256) // 32)
    want = np.stack([vals["out"][h // 12] * dims for h in range(24)])
    got = oracle.attn_row(cache, q, ids, 1 / 16)
    assert np.allclose(got, want, rtol=1e-6, atol=0), (got[0, :2], got[12, :2])
    # padding and order do not matter; the brute-force routine agrees
    got2 = oracle.attn_row(cache, q, np.array([3, -1, 1, 0, 2], np.int32), 1 / 16)
    assert np.allclose(got2, want, rtol=1e-6, atol=0)
    assert np.allclose(oracle.dense_attn_row(cache, 4, q, 1 / 16), want, rtol=1e-6, atol=0)
    # two pieces {0, 1}, {2, 3}: the hand-worked m, l and o of each
    m, l, o = oracle.partials_row(cache, q, ids, 2, 1 / 16)
    for h in range(24):
        p = pieces[h // 12]
        assert np.allclose(m[h], p["m"], rtol=0, atol=1e-6), (h, m[h])
        assert np.allclose(l[h], p["l"], rtol=1e-6, atol=0), (h, l[h])
        assert np.allclose(o[h], p["o"][:, None] * dims[None, :], rtol=1e-6, atol=1e-12), h
    assert np.allclose(oracle.merge_row(m, l, o), want, rtol=1e-6, atol=0)


def load_gate_golden():
    vals = {}
    with open(os.path.join(GOLDEN, "gate_hand.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            head, body = [p.strip() for p in line.split("|", 1)]
            vals[head] = np.array([float(t) for t in body.split()])
    return vals["gate"], vals["factor"]


def check_gate_golden():
    # out * sigmoid(g) at hand-worked points (1/2, 3/4, 1/4, 9/10, 1/10, 4/5, 1, ~0)
    g, factor = load_gate_golden()
    cache, q, vals, _ = softmax_golden_case()
    ids = np.arange(4, dtype=np.int32)
    idx = (np.arange(24)[:, None] + np.arange(256)[None, :]) % 8
    gate = g[idx].astype(np.float32)
    base = oracle.attn_row(cache, q, ids, 1 / 16)
    dims = 2.0 ** -(np.arange(256) // 32)
    want = np.stack([vals["out"][h // 12] * dims for h in range(24)]) * factor[idx]
    got = oracle.gate_row(base, gate)
    assert np.allclose(got, want, rtol=1e-6, atol=1e-20), (got[0, :4], want[0, :4])
    assert abs(got[0, 1] - 22.5) <= 1e-5
    # the whole step with the gate equals the ungated step times the gate
    wl = synth.make_workload(0, cells=200)
    wl.top_k = 64
    gate2 = (synth.Stream(83, "gate").normal(wl.rows * 24 * 256) * 3).astype(np.float32).reshape(wl.rows, 24, 256)
    plain, ids0, _ = oracle.rows(wl, threads=2)
    gated, ids1, _ = oracle.rows(wl, threads=2, gate=gate2)
    assert np.array_equal(ids0, ids1)
    assert np.allclose(gated[0], plain[0] / (1.0 + np.exp(-gate2[0].astype(np.float64))), rtol=1e-14, atol=0)


def check_dense_equivalence():
    # top_k >= visible: the whole step equals brute-force softmax over every visible cell
    wl = synth.make_workload(0, cells=96)
    wl.top_k = 128
    out, ids, _ = oracle.rows(wl, threads=2)
    assert np.array_equal(ids[0, :96], np.arange(96)) and np.all(ids[0, 96:] == -1)
    dense = oracle.dense_attn_row(wl.cache, wl.vis0(), wl.q[0], wl.scale)
    assert np.allclose(out[0], dense, rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- merge

def check_merge_golden():
    with open(os.path.join(GOLDEN, "merge_hand.txt")) as f:
        lines = [ln for ln in f if ln.startswith("case ")]
    assert len(lines) == 4
    for ln in lines:
        parts = [p.strip() for p in ln.split("|")]
        m = np.array([float(t) for t in parts[1].split()[1:]])
        l = np.array([float(t) for t in parts[2].split()[1:]])
        o = np.array([float(t) for t in parts[3].split()[1:]])
        out = float(parts[4].split()[1])
        ns = m.size
        scale = np.arange(1, 257, dtype=np.float64)
        M = np.tile(m, (24, 1))
        Lm = np.tile(l, (24, 1))
        O = np.tile(o[None, :, None] * scale[None, None, :], (24, 1, 1))
        got = oracle.merge_row(M, Lm, O)
        assert np.allclose(got, out * scale[None, :], rtol=1e-15, atol=0), (parts[0], got[0, :3])
        assert ns == O.shape[1]


def check_merge_split_invariance():
    cache = _small_cache(71, 300)
    q, _, _ = synth.make_queries(72, 1)
    ids = np.sort(synth.Stream(73, "ids").integers(300, 300))
    ids = np.unique(ids).astype(np.int32)
    ref = oracle.attn_row(cache, q[0], ids, 1 / 16)
    for ns in (1, 2, 3, 7, 64):
        m, l, o = oracle.partials_row(cache, q[0], ids, ns, 1 / 16)
        got = oracle.merge_row(m, l, o)
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-15), ns
    # more splits than cells: empty pieces are skipped
    few = ids[:5]
    m, l, o = oracle.partials_row(cache, q[0], few, 16, 1 / 16)
    assert np.sum(l[0] == 0) == 11 and np.all(np.isneginf(m[0][l[0] == 0]))
    assert np.allclose(oracle.merge_row(m, l, o), oracle.attn_row(cache, q[0], few, 1 / 16), rtol=1e-12)


# ---------------------------------------------------------------- causal mask

def check_causal_decode():
    # row i of an n-token decode sees L - n + 1 + i cells: equal to a 1-token decode at that length
    wl = synth.make_workload(1, n=4, cells=700)
    wl.top_k = 64
    out, ids, _ = oracle.rows(wl, threads=2)
    for i in range(4):
        one = synth.make_workload(1, n=4, cells=700)
        one.top_k = 64
        one.q, one.iq, one.iw = wl.q[i:i + 1], wl.iq[i:i + 1], wl.iw[i:i + 1]
        one.rows, one.L = 1, wl.L - 4 + 1 + i
        o1, i1, _ = oracle.rows(one, threads=2)
        assert np.array_equal(i1[0], ids[i]) and np.array_equal(o1[0], out[i])
        assert ids[i].max() < one.L
    # garbage in cells the last row cannot see changes nothing
    wl2 = synth.make_workload(1, n=4, cells=700)
    wl2.top_k = 64
    wl2.cache.idx_key[wl2.L:] = np.float16(30000.0)
    out2, ids2, _ = oracle.rows(wl2, threads=2)
    assert np.array_equal(ids2, ids) and np.array_equal(out2, out)
    # a cell beyond rows 0-1's horizon but inside row 2's, aligned with row 2's first indexer head:
    # row 2 must pick it, rows 0 and 1 must not see it
    wl3 = synth.make_workload(1, n=4, cells=700)
    wl3.top_k = 64
    c = wl3.L - 2
    wl3.cache.idx_key[c] = (wl3.iq[2, 0].astype(np.float32) * 20).astype(np.float16)
    _, ids3, _ = oracle.rows(wl3, threads=2)
    assert c in ids3[2] and c not in ids3[0] and c not in ids3[1]
    for i in range(4):
        assert ids3[i].max() < wl3.L - 4 + 1 + i


def check_causal_prefill():
    # prefill row t sees pos0 + t + 1 cells: equal to a 1-token decode at that length
    wl = synth.make_workload(3, cells=600, rows=5)
    wl.top_k = 100
    out, ids, _ = oracle.rows(wl, threads=2)
    for t in range(5):
        one = synth.make_workload(1, n=1, cells=600)
        one.cache = wl.cache
        one.top_k = 100
        one.q, one.iq, one.iw = wl.q[t:t + 1], wl.iq[t:t + 1], wl.iw[t:t + 1]
        one.rows, one.L = 1, wl.pos0 + t + 1
        o1, i1, _ = oracle.rows(one, threads=1)
        assert np.array_equal(i1[0], ids[t]) and np.array_equal(o1[0], out[t])
        assert ids[t].max() <= wl.pos0 + t


ALL_CHECKS = [
    check_half_decode_exhaustive, check_float_to_half_rn, check_quantize_golden,
    check_quantize_patterns, check_cache_write_layout, check_index_score_golden,
    check_index_score_onehot, check_topk_bruteforce, check_topk_special, check_attn_single_cell,
    check_attn_uniform, check_attn_dominant, check_attn_gqa_and_groups,
    check_attn_order_and_padding, check_attn_softmax_golden, check_gate_golden, check_dense_equivalence, check_merge_golden,
    check_merge_split_invariance, check_causal_decode, check_causal_prefill,
]
