"""CUDA path against the CPU oracle on the same seeded inputs (needs a B200).

Tolerances (fixed by the workload statement):
* selected id sets are bit-exact, except that a cell may be swapped at the
  k-th boundary when its oracle score is within 1e-5 relative of the oracle's
  k-th score tau (GPU scores are fp32, the oracle's float64);
* attention outputs are within 2e-3 relative error, measured per (row, head)
  as max_d |O_gpu - O_ref| / max_d |O_ref|;
* the cache-write codes and scales, and the selection on identical fp32
  scores, are bit-exact.
"""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
OUT_TOL = 2e-3
SEL_TOL = 1e-5
SPLIT_TOL = 1e-3   # GPU against GPU with a different split of the selected list
THREADS = os.cpu_count() or 1


def dev_inputs(qsa, wl):
    cache = qsa.DeviceCache.from_host(wl.cache, DEV)
    return (cache, torch.from_numpy(wl.q).to(DEV), torch.from_numpy(wl.iq).to(DEV),
            torch.from_numpy(wl.iw).to(DEV))


def rel_err(out, ref):
    """max over (row, head) of max_d |out - ref| / max_d |ref|."""
    den = np.maximum(np.abs(ref).max(-1), 1e-30)
    return float((np.abs(out - ref).max(-1) / den).max())


def check_selection(ids, ref_ids, ref_scores, top_k):
    """Apply the boundary rule row by row; return the rows whose sets match exactly."""
    exact = []
    for r in range(ref_ids.shape[0]):
        g = ids[r]
        o = ref_ids[r]
        nv = int((o >= 0).sum())
        assert int((g >= 0).sum()) == nv, f"row {r}: {int((g >= 0).sum())} ids, oracle {nv}"
        assert np.all(g[nv:] == -1) and np.all(np.diff(g[:nv]) > 0), f"row {r}: not ascending / padded"
        gs, os_ = set(g[:nv].tolist()), set(o[:nv].tolist())
        if gs == os_:
            exact.append(r)
            continue
        tau = ref_scores[r][o[:nv]].min()
        for c in gs ^ os_:
            assert abs(ref_scores[r][c] - tau) <= SEL_TOL * abs(tau), (
                f"row {r}: cell {c} (score {ref_scores[r][c]!r}) differs beyond the boundary tau={tau!r}")
    return exact


def check_outputs(qsa, cache, q, out, ids, ref_out, ref_ids, ref_scores, rows, scale, top_k):
    exact = set(check_selection(ids, ref_ids, ref_scores, top_k))
    for i, r in enumerate(rows):
        if i in exact:
            e = rel_err(out[r], ref_out[i])
        else:  # boundary swap: run the GPU attention on the oracle's own selection
            o2 = qsa.attn(cache, q[r:r + 1].contiguous(),
                          torch.from_numpy(ref_ids[i:i + 1]).to(DEV), 1, scale)
            e = rel_err(o2.cpu().numpy()[0], ref_out[i])
        assert e <= OUT_TOL, f"row {r}: relative error {e:.3e}"
    return len(exact)


# ------------------------------------------------------------------ cache write

@pytest.mark.parametrize("pattern", ["random", "signed_zeros", "pow2", "alternating", "tiny"])
def test_cache_write_bit_exact(gpu, pattern):
    qsa = gpu
    cells, pos0, n = 40, 13, 7
    host = synth.make_cache(5, cells)
    x = synth.quantizer_patterns(17, 2 * n * 2 * 8)[pattern].reshape(2, n, 2, 256)
    key = synth.make_new_cells(18, n)[2]
    cache = qsa.DeviceCache.from_host(host, DEV)
    qsa.cache_write(cache, pos0, torch.from_numpy(np.ascontiguousarray(x[0])).to(DEV),
                    torch.from_numpy(np.ascontiguousarray(x[1])).to(DEV), torch.from_numpy(key).to(DEV))
    oracle.cache_write(host, pos0, x[0], x[1], key)
    torch.cuda.synchronize()
    assert np.array_equal(cache.k.cpu().numpy(), host.k)
    assert np.array_equal(cache.v.cpu().numpy(), host.v)
    assert np.array_equal(cache.ks.cpu().numpy().view(np.uint16), host.ks.view(np.uint16))
    assert np.array_equal(cache.vs.cpu().numpy().view(np.uint16), host.vs.view(np.uint16))
    assert np.array_equal(cache.idx_key.cpu().numpy().view(np.uint16), host.idx_key.view(np.uint16))


def test_cache_write_golden(gpu):
    """The hand-worked quantizer fixtures, through the kernel."""
    from tests import pins
    qsa = gpu
    cases = pins.load_quantize_golden()
    n = (len(cases) + 15) // 16
    x = np.zeros((n * 16, 32), np.float32)
    for i, (_, xi, _, _) in enumerate(cases):
        x[i] = xi
    cache = qsa.DeviceCache.empty(n, DEV)
    xk = torch.from_numpy(x.reshape(n, 2, 256)).to(DEV)
    qsa.cache_write(cache, 0, xk, xk, torch.zeros(n, 64, dtype=torch.float16, device=DEV))
    codes = cache.k.cpu().numpy().reshape(-1, 32)
    scales = cache.ks.cpu().numpy().view(np.uint16).reshape(-1)
    for i, (name, _, sbits, want) in enumerate(cases):
        assert int(scales[i]) == sbits, name
        assert np.array_equal(codes[i], want), name


# ------------------------------------------------------------------ index score

# rows <= 8 run the decode GEMV (mma.sync); more rows run the tcgen05 GEMM (TMA + TMEM),
# here with several 128-token blocks, ragged token and cell tails
@pytest.mark.parametrize("ncells,rows", [(1000, 8), (77, 3), (4096, 1), (333, 13), (1000, 130),
                                         (4099, 300), (64, 128), (8191, 9)])
def test_index_score(gpu, ncells, rows):
    qsa = gpu
    wl = synth.make_workload(1, n=min(rows, 8), cells=ncells)
    _, iq, iw = synth.make_queries(77, rows)
    cache = qsa.DeviceCache.from_host(wl.cache, DEV)
    sc = qsa.index_score(cache, torch.from_numpy(iq).to(DEV), torch.from_numpy(iw).to(DEV), ncells)
    torch.cuda.synchronize()
    sc = sc.cpu().numpy()[:, :ncells]
    key = wl.cache.idx_key.astype(np.float64)
    for r in range(rows):
        ref = oracle.index_scores(wl.cache.idx_key, ncells, iq[r], iw[r])
        # fp32 accumulation of 64 exact fp16 products: at most 64 ulps of the sum of |terms|
        terms = np.abs(iq[r].astype(np.float64)) @ np.abs(key).T          # [4][ncells]
        bound = 2.0 ** -18 * (iw[r].astype(np.float64) @ terms) + 1e-30
        err = np.abs(sc[r] - ref)
        assert np.all(err <= bound), (r, float((err / bound).max()))


@pytest.mark.parametrize("rows", [4, 40])
def test_index_score_duplicates_bit_equal(gpu, rows):
    qsa = gpu
    wl = synth.make_workload(4, cells=3000, rows=rows)
    cache = qsa.DeviceCache.from_host(wl.cache, DEV)
    sc = qsa.index_score(cache, torch.from_numpy(wl.iq).to(DEV), torch.from_numpy(wl.iw).to(DEV), 3000)
    sc = sc.cpu().numpy()[:, :3000]
    keys = wl.cache.idx_key.view(np.uint16)
    _, first = np.unique(keys, axis=0, return_index=True)
    inv = np.unique(keys, axis=0, return_inverse=True)[1].reshape(-1)
    assert first.size < 3000  # the workload has duplicates
    for r in range(rows):
        assert np.array_equal(sc[r], sc[r][first[inv]])


# ------------------------------------------------------------------ selection

def _topk_case(qsa, scores, vis0, k):
    rows = scores.shape[0]
    ld = (scores.shape[1] + 3) // 4 * 4
    s = np.zeros((rows, ld), np.float32)
    s[:, :scores.shape[1]] = scores
    ids = qsa.topk(torch.from_numpy(s).to(DEV), vis0, k).cpu().numpy()
    for r in range(rows):
        ref = oracle.topk(scores[r, :vis0 + r].astype(np.float64), k)
        assert np.array_equal(ids[r], ref), (r, np.setdiff1d(ids[r], ref)[:5], np.setdiff1d(ref, ids[r])[:5])


def test_topk_random(gpu):
    st = synth.Stream(101, "tk")
    _topk_case(gpu, st.normal(3 * 5003).astype(np.float32).reshape(3, 5003), 5001, 512)


def test_topk_ties(gpu):
    st = synth.Stream(102, "tk")
    s = (np.round(st.normal(2 * 20000) * 2) / 2).astype(np.float32).reshape(2, 20000)
    _topk_case(gpu, s, 19999, 2048)


@pytest.mark.parametrize("V,k", [(100, 512), (512, 512), (513, 512), (1, 1), (40, 1), (4097, 4096)])
def test_topk_sizes(gpu, V, k):
    st = synth.Stream(103 + V, "tk")
    s = st.normal(2 * (V + 1)).astype(np.float32).reshape(2, V + 1)
    _topk_case(gpu, s, V, k)


def test_topk_all_equal_and_signed_zero(gpu):
    s = np.zeros((2, 3000), np.float32)
    s[1, ::2] = -0.0
    s[1, 5] = -1e-30
    _topk_case(gpu, s, 2999, 700)


def test_topk_negative(gpu):
    st = synth.Stream(104, "tk")
    _topk_case(gpu, (-np.abs(st.normal(2 * 9000)) - 3).astype(np.float32).reshape(2, 9000), 8999, 1000)


def test_topk_candidate_overflow(gpu):
    # every score in one coarse (fp16) bin, all distinct in fp32: the candidate list
    # overflows and the final pass re-reads the row
    st = synth.Stream(105, "tk")
    V = 50000
    s = (1.0 + np.floor(st.uniform(V) * 4096) * 2.0 ** -23).astype(np.float32)[None, :]
    _topk_case(gpu, s, V, 2048)


def test_topk_threshold_bin_sizes(gpu):
    # one row per size of the threshold bin, around the limits of the one-warp
    # searches (in registers up to 1024 candidates, shared-memory digits beyond):
    # 1800 cells clearly above, the bin's cells in [10.01, 10.4] (one fp16 bin) with
    # 40 distinct values, so ties cross the CTAs' ranges, the rest far below
    st = synth.Stream(108, "tk")
    V, above, k = 60000, 1800, 2048
    sizes = [250, 512, 513, 1024, 1025, 3000]
    s = np.zeros((len(sizes), V + len(sizes)), np.float32)
    for r, nb in enumerate(sizes):
        s[r] = st.uniform(V + len(sizes), 0.0, 5.0)
        pick = np.argsort(st.uniform(V), kind="stable")[:above + nb]
        s[r, pick[:above]] = st.uniform(above, 20.0, 30.0)
        s[r, pick[above:]] = 10.01 + np.floor(st.uniform(nb) * 40) * 0.01
    _topk_case(gpu, s, V, k)


@pytest.mark.parametrize("V,ties", [(65537, False), (200000, True), (262142, False)])
def test_topk_wide_cluster(gpu, V, ties):
    # rows of 65537 .. 262144 cells: one 16-CTA cluster per row (32 cells per thread)
    st = synth.Stream(109 + V, "tk")
    s = st.normal(3 * (V + 2)).reshape(3, V + 2)
    if ties:
        s = np.round(s * 4) / 4
    _topk_case(gpu, s.astype(np.float32), V, 2048)


def test_topk_many_windows(gpu):
    st = synth.Stream(106, "tk")
    V = (1 << 19) * 2 + 777
    s = np.round(st.normal(V) * 64).astype(np.float32)[None, :]
    _topk_case(gpu, s, V, 4096)


def test_topk_max_k(gpu):
    st = synth.Stream(107, "tk")
    _topk_case(gpu, st.normal(40000).astype(np.float32)[None, :], 40000, 16384)


# ------------------------------------------------------------------ attention and merge

def _id_lists(seed, rows, cells, k, nvalid):
    st = synth.Stream(seed, "ids")
    ids = -np.ones((rows, k), np.int32)
    for r in range(rows):
        pick = np.sort(np.argsort(st.uniform(cells), kind="stable")[:nvalid[r]]).astype(np.int32)
        ids[r, :nvalid[r]] = pick
    return ids


# up to 8 rows run the 4-warp attention kernel, more rows the 2-warp one
@pytest.mark.parametrize("rows", [3, 12])
@pytest.mark.parametrize("nsplit", [1, 3, 8, 64])
def test_attn_vs_oracle(gpu, nsplit, rows):
    qsa = gpu
    cells, k = 4096, 512
    wl = synth.make_workload(0, cells=cells)
    q, _, _ = synth.make_queries(201, rows)
    ids = _id_lists(202, rows, cells, k, ([512, 300, 17] * 4)[:rows])
    cache = qsa.DeviceCache.from_host(wl.cache, DEV)
    qd = torch.from_numpy(q).to(DEV)
    idd = torch.from_numpy(ids).to(DEV)
    res = qsa.attn(cache, qd, idd, nsplit, 1 / 16)
    out = res if nsplit == 1 else qsa.merge(res)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    for r in range(rows):
        ref = oracle.attn_row(wl.cache, q[r], ids[r], 1 / 16)
        assert rel_err(out[r], ref) <= OUT_TOL
    if nsplit > 1:
        part = res.cpu().numpy()
        for r in range(rows):
            m, l, o = oracle.partials_row(wl.cache, q[r], ids[r], nsplit, 1 / 16)
            pm, pl, po = part[r, :, :, 0], part[r, :, :, 1], part[r, :, :, 2:].astype(np.float64)
            empty = l == 0
            assert np.array_equal(pl == 0, empty) and np.all(np.isneginf(pm[empty]))
            assert np.all(po[empty] == 0)
            full = ~empty
            # the piece maximum (natural-log units), its sum of weights, and its own output o / l
            assert np.all(np.abs(pm[full] - m[full]) <= 2e-3)
            assert np.allclose(pl[full] * np.exp(pm[full] - m[full]), l[full], rtol=5e-3)
            assert rel_err(po[full] / pl[full][:, None], o[full] / l[full][:, None]) <= OUT_TOL


def _check_attn(qsa, cache_h, cache, q, ids, nsplit, scale=1 / 16):
    res = qsa.attn(cache, torch.from_numpy(q).to(DEV), torch.from_numpy(ids).to(DEV), nsplit, scale)
    out = (res if nsplit == 1 else qsa.merge(res)).cpu().numpy()
    for r in range(q.shape[0]):
        assert rel_err(out[r], oracle.attn_row(cache_h, q[r], ids[r], scale)) <= OUT_TOL, f"row {r}"
    return res


# more than 8 rows (the prompt-chunk kernel): ragged last blocks, rows with one or
# no cell, splits past the end of the list
@pytest.mark.parametrize("rows,k,nsplit", [(9, 200, 1), (16, 129, 1), (10, 100, 64), (33, 2048, 3)])
def test_attn_many_rows_shapes(gpu, rows, k, nsplit):
    qsa = gpu
    cells = 4096
    wl = synth.make_workload(0, cells=cells)
    q, _, _ = synth.make_queries(211, rows)
    nvalid = [k, 1, 0] + [(k * (r + 1)) // rows for r in range(rows - 3)]
    ids = _id_lists(212, rows, cells, k, nvalid)
    cache = qsa.DeviceCache.from_host(wl.cache, DEV)
    res = _check_attn(qsa, wl.cache, cache, q, ids, nsplit)
    if nsplit > 1:
        part = res.cpu().numpy()
        empty = part[:, :, :, 1] == 0
        assert np.all(np.isneginf(part[:, :, :, 0][empty])) and np.all(part[:, :, :, 2:][empty] == 0)
        assert np.all(empty[2])  # the row without cells


def test_attn_rising_maxima(gpu):
    """Cells listed by ascending logit, so the running maximum keeps moving (by more
    than 2^8 between the first and the last 128 cells) and the accumulated output
    is rescaled many times."""
    qsa = gpu
    rows, cells, k = 9, 4096, 1024
    cache_h = synth.make_cache(214, cells)
    q, _, _ = synth.make_queries(215, rows)
    q *= 2
    kd = cache_h.k.astype(np.float64) * np.repeat(cache_h.ks.astype(np.float64), 32, -1)
    ids = np.empty((rows, k), np.int32)
    for r in range(rows):
        logit = kd[:, 0, :] @ q[r, r % 12].astype(np.float64) / 16
        order = np.argsort(logit, kind="stable")
        ids[r] = order[::cells // k][:k]
        # log2-domain maxima of the 128-cell tiles: the last one is far above the first
        tmax = (logit[ids[r]] / np.log(2)).reshape(-1, 128).max(1)
        assert tmax[-1] - tmax[0] > 8 + 1
    _check_attn(qsa, cache_h, qsa.DeviceCache.from_host(cache_h, DEV), q, ids, 1)
    _check_attn(qsa, cache_h, qsa.DeviceCache.from_host(cache_h, DEV), q, ids, 5)


def test_attn_small_v_scales(gpu):
    qsa = gpu
    cells = 2000
    cache_h = synth.make_cache(203, cells, vs_range=(1e-4, 0.05))
    q, _, _ = synth.make_queries(204, 2)
    ids = _id_lists(205, 2, cells, 2048, [2000, 1999])
    cache = qsa.DeviceCache.from_host(cache_h, DEV)
    out = qsa.attn(cache, torch.from_numpy(q).to(DEV), torch.from_numpy(ids).to(DEV), 1, 1 / 16).cpu().numpy()
    for r in range(2):
        assert rel_err(out[r], oracle.attn_row(cache_h, q[r], ids[r], 1 / 16)) <= OUT_TOL


def test_attn_single_and_empty(gpu):
    qsa = gpu
    cache_h = synth.make_cache(206, 64)
    q, _, _ = synth.make_queries(207, 2)
    ids = -np.ones((2, 40), np.int32)
    ids[0, 0] = 37  # one cell: O = its dequantised V row
    cache = qsa.DeviceCache.from_host(cache_h, DEV)
    out = qsa.attn(cache, torch.from_numpy(q).to(DEV), torch.from_numpy(ids).to(DEV), 1).cpu().numpy()
    vd = cache_h.v[37].astype(np.float64) * np.repeat(cache_h.vs[37].astype(np.float64), 32, -1)
    for h in range(24):
        assert np.allclose(out[0, h], vd[h // 12], rtol=1e-3, atol=0)
    assert np.all(out[1] == 0)  # no cells at all
    part = qsa.attn(cache, torch.from_numpy(q).to(DEV), torch.from_numpy(ids).to(DEV), 4).cpu().numpy()
    assert np.all(np.isneginf(part[1, :, :, 0])) and np.all(part[1, :, :, 1:] == 0)


@pytest.mark.parametrize("rows,k", [(9, 1), (12, 300), (17, 4096)])
def test_attn_prompt_kernel_edges(gpu, rows, k):
    # more than 8 rows in one piece (the prompt-chunk kernel): lists shorter than one
    # 32-cell block, ragged last blocks, an empty row, ids past the cache as empty slots,
    # a query head of zeros (equal weights), the output gate in the epilogue
    qsa = gpu
    cells = 5000
    cache_h = synth.make_cache(231, cells)
    q, _, _ = synth.make_queries(232, rows)
    q[2, 5] = 0.0
    nvalid = [k, 0] + [max(1, (k * (r + 1)) // rows) for r in range(rows - 2)]
    ids = _id_lists(233, rows, cells, k, nvalid)
    if k > 1:
        ids[0, -1] = cells + 7
    gate = _gate(234, rows)
    cache = qsa.DeviceCache.from_host(cache_h, DEV)
    out = qsa.attn(cache, torch.from_numpy(q).to(DEV), torch.from_numpy(ids).to(DEV), 1, 1 / 16,
                   gate=gate).cpu().numpy()
    g = gate.cpu().numpy()
    assert np.all(out[1] == 0)  # no cells at all
    for r in [0] + list(range(2, rows)):
        ids_r = np.where((ids[r] >= 0) & (ids[r] < cells), ids[r], -1).astype(np.int32)
        ref = oracle.gate_row(oracle.attn_row(cache_h, q[r], ids_r, 1 / 16), g[r])
        assert rel_err(out[r], ref) <= OUT_TOL, f"row {r}"


def test_attn_prompt_kernel_golden(gpu):
    # the hand-worked softmax fixture as ten rows of one call (the prompt-chunk kernel)
    from tests import pins
    qsa = gpu
    cache_h, q, vals, _ = pins.softmax_golden_case()
    cache = qsa.DeviceCache.from_host(cache_h, DEV)
    dims = 2.0 ** -(np.arange(256) // 32)
    want = np.stack([vals["out"][h // 12] * dims for h in range(24)])
    ids = torch.arange(4, dtype=torch.int32, device=DEV)[None].repeat(10, 1)
    qd = torch.from_numpy(np.repeat(q[None], 10, 0)).to(DEV)
    out = qsa.attn(cache, qd, ids, 1, 1 / 16).cpu().numpy()
    for r in range(10):
        assert rel_err(out[r], want) <= OUT_TOL


@pytest.mark.parametrize("rows,nsplit", [(3, 1), (3, 8), (12, 1)])
def test_attn_query_offset(gpu, rows, nsplit):
    # queries with a common offset of 2 standard deviations: the K codes enter the tiles as
    # 1152 + code and each group's accumulator starts at -1152 times its query sum, so the
    # cancellation is large here (both the decode and the prompt-chunk kernels).  Larger offsets
    # take every variant past the tolerance through the fp16 rounding of q and P alone.
    qsa = gpu
    cells, k = 3000, 700
    cache_h = synth.make_cache(241, cells)
    q, _, _ = synth.make_queries(242, rows)
    q = (q + 2.0).astype(np.float32)
    q[0, 3] = -q[0, 3]  # one head with the opposite offset
    ids = _id_lists(243, rows, cells, k, [k] * rows)
    _check_attn(qsa, cache_h, qsa.DeviceCache.from_host(cache_h, DEV), q, ids, nsplit)


def test_merge_vs_oracle(gpu):
    qsa = gpu
    st = synth.Stream(301, "merge")
    rows, ns = 3, 64
    m = st.normal(rows * 24 * ns).reshape(rows, 24, ns) * 3
    l = st.uniform(rows * 24 * ns, 0.5, 100).reshape(rows, 24, ns)
    o = st.normal(rows * 24 * ns * 256).reshape(rows, 24, ns, 256) * 10
    empty = st.uniform(rows * 24 * ns).reshape(rows, 24, ns) < 0.2
    m[empty], l[empty], o[empty] = -np.inf, 0, 0
    part = np.concatenate([m[..., None], l[..., None], o], -1).astype(np.float32)
    out = qsa.merge(torch.from_numpy(part).to(DEV)).cpu().numpy()
    for r in range(rows):
        ref = oracle.merge_row(part[r, :, :, 0].astype(np.float64), part[r, :, :, 1].astype(np.float64),
                               part[r, :, :, 2:].astype(np.float64))
        assert rel_err(out[r], ref) <= 1e-5


def test_merge_golden(gpu):
    qsa = gpu
    from tests import pins
    import os as _os
    lines = [ln for ln in open(_os.path.join(pins.GOLDEN, "merge_hand.txt")) if ln.startswith("case ")]
    for ln in lines:
        parts = [p.strip() for p in ln.split("|")]
        m = np.array([float(t) for t in parts[1].split()[1:]])
        l = np.array([float(t) for t in parts[2].split()[1:]])
        o = np.array([float(t) for t in parts[3].split()[1:]])
        want = float(parts[4].split()[1])
        ns = m.size
        part = np.zeros((1, 24, ns, 258), np.float32)
        part[0, :, :, 0], part[0, :, :, 1] = m, l
        part[0, :, :, 2:] = o[None, :, None] * np.arange(1, 257)[None, None, :]
        out = qsa.merge(torch.from_numpy(part).to(DEV)).cpu().numpy()
        assert np.allclose(out[0], want * np.arange(1, 257)[None, :], rtol=2e-6), parts[0]


# ------------------------------------------------------------------ the whole step

def _decode_case(qsa, wl, nsplit=None):
    cache, q, iq, iw = dev_inputs(qsa, wl)
    ids = torch.empty(wl.rows, wl.top_k, dtype=torch.int32, device=DEV)
    ns = wl.nsplit if nsplit is None else nsplit
    out = qsa.decode(cache, wl.L, q, iq, iw, wl.top_k, ns, wl.scale, ids_out=ids)
    torch.cuda.synchronize()
    ref_out, ref_ids, ref_sc = oracle.rows(wl, want_scores=True, threads=THREADS)
    return check_outputs(qsa, cache, q, out.cpu().numpy(), ids.cpu().numpy(), ref_out, ref_ids, ref_sc,
                         list(range(wl.rows)), wl.scale, wl.top_k)


def test_decode_config0(gpu):
    assert _decode_case(gpu, synth.make_workload(0)) >= 0


@pytest.mark.parametrize("nsplit", [1, 8])
def test_decode_config0_splits(gpu, nsplit):
    _decode_case(gpu, synth.make_workload(0), nsplit)


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 6, 7, 8])
def test_decode_config1(gpu, n):
    _decode_case(gpu, synth.make_workload(1, n=n))


@pytest.mark.parametrize("n", [1, 3])
def test_decode_long_rows_auto_split(gpu, n):
    # rows of more than 65536 cells with the automatic split: one 16-CTA selection cluster
    # per row, then 32 pieces of attention and their merge
    wl = synth.make_workload(2, n=n)
    wl.nsplit = 0
    _decode_case(gpu, wl)


def test_decode_config2(gpu):
    _decode_case(gpu, synth.make_workload(2))


@pytest.mark.parametrize("n", [1, 2, 4, 8])
@pytest.mark.parametrize("pos0", [0, 1, 63, 64, 511, 512, 513, 2047, 2048, 2050, 8192, 30000])
def test_decode_boundary_grid(gpu, pos0, n):
    # n new cells after pos0 cached ones: token i sees pos0 + 1 + i cells, from a single cell to
    # well past top_k = 2048 (the dense path up to 2048 visible cells, scores and selection beyond)
    _decode_case(gpu, synth.make_workload(1, n=n, cells=pos0 + n), 0)


def test_decode_small_ragged(gpu):
    wl = synth.make_workload(1, n=5, cells=2077)
    wl.top_k = 300
    _decode_case(gpu, wl, 7)


def test_decode_dense_when_few_cells(gpu):
    # every row sees fewer cells than top_k: all visible cells, equal to brute-force softmax
    qsa = gpu
    wl = synth.make_workload(1, n=4, cells=300)
    wl.top_k = 512
    cache, q, iq, iw = dev_inputs(qsa, wl)
    ids = torch.empty(4, 512, dtype=torch.int32, device=DEV)
    out = qsa.decode(cache, wl.L, q, iq, iw, 512, 0, wl.scale, ids_out=ids).cpu().numpy()
    ids = ids.cpu().numpy()
    for i in range(4):
        V = wl.L - 4 + 1 + i
        assert np.array_equal(ids[i, :V], np.arange(V)) and np.all(ids[i, V:] == -1)
        assert rel_err(out[i], oracle.dense_attn_row(wl.cache, V, wl.q[i], wl.scale)) <= OUT_TOL


@pytest.mark.parametrize("n,nsplit", [(1, 1), (3, 5), (8, 32), (8, 0)])
def test_decode_short_context_bit_equal(gpu, n, nsplit):
    # every row sees at most top_k cells: the step skips the scores and the selection and
    # walks cells 0 .. V - 1 itself, bit-equal to the selection's list run by qsa_attn
    qsa = gpu
    top_k = 512
    wl = synth.make_workload(1, n=n, cells=top_k)
    cache, q, iq, iw = dev_inputs(qsa, wl)
    ids = torch.full((n, top_k), 7, dtype=torch.int32, device=DEV)
    out = qsa.decode(cache, wl.L, q, iq, iw, top_k, nsplit, wl.scale, ids_out=ids).cpu().numpy()
    ns = nsplit or qsa_auto_nsplit(n, top_k)
    ref_ids = -np.ones((n, top_k), np.int32)
    for i in range(n):
        ref_ids[i, :wl.L - n + 1 + i] = np.arange(wl.L - n + 1 + i)
    assert np.array_equal(ids.cpu().numpy(), ref_ids)
    res = qsa.attn(cache, q, torch.from_numpy(ref_ids).to(DEV), ns, wl.scale)
    two = (res if ns == 1 else qsa.merge(res)).cpu().numpy()
    assert np.array_equal(out.view(np.uint32), two.view(np.uint32))
    for i in range(n):
        assert rel_err(out[i], oracle.dense_attn_row(wl.cache, wl.L - n + 1 + i, wl.q[i], wl.scale)) <= OUT_TOL


@pytest.mark.parametrize("extra", [0, 1])
def test_decode_short_context_boundary(gpu, extra):
    # the last row sees top_k cells (implicit list) or top_k + 1 (scores and selection)
    wl = synth.make_workload(1, n=4, cells=300 + extra)
    wl.top_k = 300
    _decode_case(gpu, wl, 3)


@pytest.mark.parametrize("T", [4, 16])
def test_prefill_short_context(gpu, T):
    # a chunk inside the first top_k cells: every row attends to all the cells it sees
    qsa = gpu
    top_k, pos0 = 512, 100
    wl = synth.make_workload(3, cells=pos0 + T, rows=T)
    cache, q, iq, iw = dev_inputs(qsa, wl)
    ids = torch.empty(T, top_k, dtype=torch.int32, device=DEV)
    out = qsa.prefill_chunk(cache, pos0, q, iq, iw, top_k, wl.scale, ids_out=ids).cpu().numpy()
    ids = ids.cpu().numpy()
    for t in range(T):
        V = pos0 + t + 1
        assert np.array_equal(ids[t, :V], np.arange(V)) and np.all(ids[t, V:] == -1)
        assert rel_err(out[t], oracle.dense_attn_row(wl.cache, V, wl.q[t], wl.scale)) <= OUT_TOL


def qsa_auto_nsplit(rows, top_k):
    import bench
    return bench.auto_nsplit(rows, top_k)


def test_decode_nsplit_invariance(gpu):
    qsa = gpu
    wl = synth.make_workload(1, n=2, cells=6000)
    cache, q, iq, iw = dev_inputs(qsa, wl)
    outs, idss = [], []
    for ns in (1, 2, 7, 64, 0):  # 0: the automatic split
        ids = torch.empty(2, wl.top_k, dtype=torch.int32, device=DEV)
        outs.append(qsa.decode(cache, wl.L, q, iq, iw, wl.top_k, ns, wl.scale, ids_out=ids).cpu().numpy())
        idss.append(ids.cpu().numpy())
    # Q and the softmax weights P are rounded to fp16 relative to each piece's own
    # running maximum, so split counts differ by that rounding (~2^-12 relative per
    # weight), well inside the parity tolerance each of them meets against the oracle.
    for o, i in zip(outs[1:], idss[1:]):
        assert np.array_equal(i, idss[0])
        assert rel_err(o, outs[0]) <= SPLIT_TOL


def _prefill_case(qsa, wl, rows, batch=256):
    """One GPU chunk; the oracle on the given rows, `batch` rows at a time (its float64
    scores of a batch are held at once)."""
    cache, q, iq, iw = dev_inputs(qsa, wl)
    ids = torch.empty(wl.rows, wl.top_k, dtype=torch.int32, device=DEV)
    out = qsa.prefill_chunk(cache, wl.pos0, q, iq, iw, wl.top_k, wl.scale, ids_out=ids)
    torch.cuda.synchronize()
    out, ids = out.cpu().numpy(), ids.cpu().numpy()
    exact = 0
    for b in range(0, len(rows), batch):
        part = rows[b:b + batch]
        ref_out, ref_ids, ref_sc = oracle.rows(wl, np.array(part), want_scores=True, threads=THREADS)
        exact += check_outputs(qsa, cache, q, out, ids[part], ref_out, ref_ids, ref_sc, part, wl.scale,
                               wl.top_k)
    return exact


def test_prefill_small_all_rows(gpu):
    wl = synth.make_workload(3, cells=2500, rows=150)
    wl.top_k = 256
    _prefill_case(gpu, wl, list(range(150)))


def test_prefill_config3_all_rows(gpu):
    # T = 2048 at 63488 over 65536 cells: every row, so every 128-token GEMM tile and every
    # row's selection is compared with the oracle (about 1.3e8 cells of float64 scores)
    wl = synth.make_workload(3)
    _prefill_case(gpu, wl, list(range(wl.rows)))


def test_prefill_config4_all_rows(gpu):
    # T = 1024 at 261120 over 262144 cells with 10% duplicated keys (ties): every row
    wl = synth.make_workload(4)
    _prefill_case(gpu, wl, list(range(wl.rows)))


@pytest.mark.parametrize("T,cells,top_k", [(9, 1500, 128), (65, 3000, 512), (200, 9000, 2048)])
def test_prefill_ragged_chunks(gpu, T, cells, top_k):
    # chunks just above 8 rows (the GEMV/cluster path ends there), a token block and one
    # row, cell counts that are not multiples of the 128-cell tiles
    wl = synth.make_workload(3, cells=cells, rows=T)
    wl.top_k = top_k
    _prefill_case(gpu, wl, list(range(T)))


def test_prefill_sample_fooled(gpu):
    # every 16th cell (the cells the threshold pass samples) has a large key and the rest
    # small ones: the sampled threshold admits fewer than top_k cells, so every row takes
    # the exact recomputing path
    wl = synth.make_workload(3, cells=6000, rows=40)
    wl.top_k = 512
    key = wl.cache.idx_key.astype(np.float32)
    key *= 0.05
    key[::16] *= 400.0
    wl.cache.idx_key = key.astype(np.float16)
    _prefill_case(gpu, wl, list(range(40)))


def test_prefill_all_keys_equal(gpu):
    # identical keys: every visible cell ties, the candidate lists overflow and the exact
    # path keeps the lowest indices
    wl = synth.make_workload(3, cells=5000, rows=30)
    wl.top_k = 700
    wl.cache.idx_key[:] = wl.cache.idx_key[0]
    qsa = gpu
    cache, q, iq, iw = dev_inputs(qsa, wl)
    ids = torch.empty(30, 700, dtype=torch.int32, device=DEV)
    qsa.prefill_chunk(cache, wl.pos0, q, iq, iw, 700, wl.scale, ids_out=ids)
    assert np.array_equal(ids.cpu().numpy(), np.tile(np.arange(700, dtype=np.int32), (30, 1)))


def test_prefill_row_equals_decode(gpu):
    # prefill row t is a one-token decode at L = pos0 + t + 1.  The two paths score on
    # different tensor-core instructions (tcgen05 GEMM vs mma.sync GEMV), so their fp32
    # scores may differ in the last bits: the id sets must agree up to the boundary rule.
    qsa = gpu
    wl = synth.make_workload(3, cells=3000, rows=64)
    wl.top_k = 512
    cache, q, iq, iw = dev_inputs(qsa, wl)
    ids_p = torch.empty(64, 512, dtype=torch.int32, device=DEV)
    out_p = qsa.prefill_chunk(cache, wl.pos0, q, iq, iw, 512, wl.scale, ids_out=ids_p)
    rows = [0, 31, 63]
    _, ref_ids, ref_sc = oracle.rows(wl, np.array(rows), want_scores=True, threads=THREADS)
    for i, t in enumerate(rows):
        ids_d = torch.empty(1, 512, dtype=torch.int32, device=DEV)
        out_d = qsa.decode(cache, wl.pos0 + t + 1, q[t:t + 1], iq[t:t + 1], iw[t:t + 1], 512, 1, wl.scale,
                           ids_out=ids_d)
        a, b = ids_d[0].cpu().numpy(), ids_p[t].cpu().numpy()
        check_selection(a[None], ref_ids[i:i + 1], ref_sc[i:i + 1], 512)
        check_selection(b[None], ref_ids[i:i + 1], ref_sc[i:i + 1], 512)
        if np.array_equal(a, b):
            # prefill picks its own split count; see test_decode_nsplit_invariance
            assert rel_err(out_d.cpu().numpy()[0], out_p.cpu().numpy()[t]) <= SPLIT_TOL


def test_attn_softmax_golden(gpu):
    # the hand-worked softmax fixture through the kernels: weights w_c / sum(w) from
    # logits ln w_c, outputs 30 and 19.2 (times 2^-(d div 32)), one piece and two pieces
    from tests import pins
    qsa = gpu
    cache_h, q, vals, _ = pins.softmax_golden_case()
    cache = qsa.DeviceCache.from_host(cache_h, DEV)
    dims = 2.0 ** -(np.arange(256) // 32)
    want = np.stack([vals["out"][h // 12] * dims for h in range(24)])
    ids = torch.arange(4, dtype=torch.int32, device=DEV)[None]
    qd = torch.from_numpy(q[None]).to(DEV)
    one = qsa.attn(cache, qd, ids, 1, 1 / 16).cpu().numpy()[0]
    two = qsa.merge(qsa.attn(cache, qd, ids, 2, 1 / 16)).cpu().numpy()[0]
    assert rel_err(one, want) <= OUT_TOL and rel_err(two, want) <= OUT_TOL


def _gate(seed, rows):
    return torch.from_numpy((synth.Stream(seed, "gate").normal(rows * 24 * 256) * 2).astype(np.float32)
                            .reshape(rows, 24, 256)).to(DEV)


@pytest.mark.parametrize("nsplit", [1, 6])
def test_attn_and_merge_gate(gpu, nsplit):
    # out = O * sigmoid(gate): nsplit 1 gates in the attention epilogue, more pieces in the merge
    qsa = gpu
    rows, cells, k = 3, 3000, 256
    wl = synth.make_workload(0, cells=cells)
    q, _, _ = synth.make_queries(221, rows)
    ids = _id_lists(222, rows, cells, k, [256, 100, 1])
    gate = _gate(223, rows)
    cache = qsa.DeviceCache.from_host(wl.cache, DEV)
    qd, idd = torch.from_numpy(q).to(DEV), torch.from_numpy(ids).to(DEV)
    if nsplit == 1:
        out = qsa.attn(cache, qd, idd, 1, 1 / 16, gate=gate)
        plain = qsa.attn(cache, qd, idd, 1, 1 / 16)
    else:
        part = qsa.attn(cache, qd, idd, nsplit, 1 / 16)
        out, plain = qsa.merge(part, gate=gate), qsa.merge(part)
    out, plain, g = out.cpu().numpy(), plain.cpu().numpy(), gate.cpu().numpy()
    for r in range(rows):
        ref = oracle.gate_row(oracle.attn_row(wl.cache, q[r], ids[r], 1 / 16), g[r])
        assert rel_err(out[r], ref) <= OUT_TOL
        assert np.allclose(out[r], plain[r] / (1 + np.exp(-g[r].astype(np.float64))), rtol=1e-5, atol=1e-30)


@pytest.mark.parametrize("kind", ["decode", "decode_dense", "prefill"])
def test_step_with_append_and_gate(gpu, kind):
    # one call appends the rows' own cells (quantized exactly as qsa_cache_write does), then
    # runs the step and gates the output; bit-equal to a separate cache write plus the step.
    # Decode appends inside its scoring kernel; the short-context path and prefill chunks
    # run the cache write first.
    qsa = gpu
    if kind.startswith("decode"):
        wl = synth.make_workload(1, n=6, cells=7000 if kind == "decode" else 400)
        if kind == "decode_dense":
            wl.top_k = 512
        pos = wl.L - wl.rows
    else:
        wl = synth.make_workload(3, cells=2600, rows=140)
        wl.top_k = 256
        pos = wl.pos0
    rows = wl.rows
    kn, vn, keyn = synth.make_new_cells(231, rows)
    gate = _gate(232, rows)
    cache, q, iq, iw = dev_inputs(qsa, wl)       # the new cells' slots hold other data
    twin, _, _, _ = dev_inputs(qsa, wl)
    app = (torch.from_numpy(kn).to(DEV), torch.from_numpy(vn).to(DEV), torch.from_numpy(keyn).to(DEV))
    ids = torch.empty(rows, wl.top_k, dtype=torch.int32, device=DEV)
    ids2 = torch.empty_like(ids)
    if kind.startswith("decode"):
        out = qsa.decode(cache, wl.L, q, iq, iw, wl.top_k, 0, wl.scale, ids_out=ids, append=app, gate=gate)
        qsa.cache_write(twin, pos, *app)
        out2 = qsa.decode(twin, wl.L, q, iq, iw, wl.top_k, 0, wl.scale, ids_out=ids2, gate=gate)
    else:
        out = qsa.prefill_chunk(cache, pos, q, iq, iw, wl.top_k, wl.scale, ids_out=ids, append=app, gate=gate)
        qsa.cache_write(twin, pos, *app)
        out2 = qsa.prefill_chunk(twin, pos, q, iq, iw, wl.top_k, wl.scale, ids_out=ids2, gate=gate)
    torch.cuda.synchronize()
    for a, b in ((cache.k, twin.k), (cache.v, twin.v), (cache.ks, twin.ks), (cache.vs, twin.vs),
                 (cache.idx_key, twin.idx_key)):
        assert torch.equal(a, b)
    assert torch.equal(ids, ids2)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), out2.cpu().numpy().view(np.uint32))
    # against the oracle: its own cache write, then the gated step
    oracle.cache_write(wl.cache, pos, kn, vn, keyn)
    assert np.array_equal(cache.k.cpu().numpy(), wl.cache.k)
    sel = list(range(0, rows, max(1, rows // 10)))
    ref_out, ref_ids, ref_sc = oracle.rows(wl, np.array(sel), want_scores=True, threads=THREADS,
                                           gate=gate.cpu().numpy())
    exact = set(check_selection(ids.cpu().numpy()[sel], ref_ids, ref_sc, wl.top_k))
    out = out.cpu().numpy()
    g = gate.cpu().numpy()
    for i, r in enumerate(sel):
        if i in exact:
            got = out[r]
        else:
            got = qsa.attn(cache, q[r:r + 1].contiguous(), torch.from_numpy(ref_ids[i:i + 1]).to(DEV), 1,
                           wl.scale, gate=gate[r:r + 1].contiguous()).cpu().numpy()[0]
        assert rel_err(got, ref_out[i]) <= OUT_TOL, r


SENTINEL = 0x7FC0BEEF  # a NaN bit pattern no kernel writes


def _guarded(shape, dtype, pad):
    """A buffer of `shape` with `pad` guard elements before and after it, all set to the
    sentinel bits; returns (whole buffer, the view handed to the library)."""
    n = int(np.prod(shape))
    whole = torch.full((n + 2 * pad,), SENTINEL, dtype=torch.int32, device=DEV)
    whole = whole.view(dtype) if dtype != torch.int32 else whole
    return whole, whole[pad:pad + n].view(*shape)


def _guards_intact(whole, pad):
    bits = whole.view(torch.int32).cpu().numpy()
    return bool(np.all(bits[:pad] == SENTINEL) and np.all(bits[-pad:] == SENTINEL))


@pytest.mark.parametrize("kind", ["decode", "prefill"])
def test_step_writes_stay_inside_outputs(gpu, kind):
    # out, ids_out and the workspace each sit between guard regions (a whole row of out
    # on both sides, 64 ids, 4 KB of workspace): the step must write only inside them
    qsa = gpu
    if kind == "decode":
        wl = synth.make_workload(1, n=5, cells=9000)
        mode, L = qsa.MODE_DECODE, wl.L
    else:
        wl = synth.make_workload(3, cells=2600, rows=140)
        wl.top_k = 256
        mode, L = qsa.MODE_PREFILL, wl.pos0 + wl.rows
    cache, q, iq, iw = dev_inputs(qsa, wl)
    rows = wl.rows
    pad_out, pad_ids, pad_ws = 24 * 256, 64, 1024
    out_w, out = _guarded((rows, 24, 256), torch.float32, pad_out)
    ids_w, ids = _guarded((rows, wl.top_k), torch.int32, pad_ids)
    nbytes = qsa.workspace_bytes(mode, rows, L, wl.top_k, wl.nsplit if kind == "decode" else 0)
    ws_w, ws = _guarded(((nbytes + 3) // 4,), torch.int32, pad_ws)
    ws = ws.view(torch.uint8)
    if kind == "decode":
        qsa.decode(cache, wl.L, q, iq, iw, wl.top_k, wl.nsplit, wl.scale, ws=ws, out=out, ids_out=ids)
    else:
        qsa.prefill_chunk(cache, wl.pos0, q, iq, iw, wl.top_k, wl.scale, ws=ws, out=out, ids_out=ids)
    torch.cuda.synchronize()
    assert _guards_intact(out_w, pad_out) and _guards_intact(ids_w, pad_ids) and _guards_intact(ws_w, pad_ws)
    # and the result inside is the step's result
    sel = list(range(0, rows, max(1, rows // 12)))
    ref_out, ref_ids, ref_sc = oracle.rows(wl, np.array(sel), want_scores=True, threads=THREADS)
    check_outputs(qsa, cache, q, out.cpu().numpy(), ids.cpu().numpy()[sel], ref_out, ref_ids, ref_sc, sel,
                  wl.scale, wl.top_k)


def test_errors_and_launch_count(gpu):
    qsa = gpu
    wl = synth.make_workload(0, cells=500)
    cache, q, iq, iw = dev_inputs(qsa, wl)
    small = qsa.workspace(64, DEV)
    before = qsa.launch_count()
    with pytest.raises(qsa.QSAError) as e:
        qsa.decode(cache, wl.L, q, iq, iw, wl.top_k, 0, wl.scale, ws=small)
    assert e.value.code == 2 and qsa.launch_count() == before
    qsa.decode(cache, wl.L, q, iq, iw, wl.top_k, 0, wl.scale)
    assert qsa.launch_count() > before


def test_bounded_wait_reports_timeout(gpu):
    """A kernel waiting on a barrier nothing completes gives up after about one
    second and records QSA_ERR_TIMEOUT; the context keeps working afterwards."""
    qsa = gpu
    assert qsa.device_status() == 0
    qsa.selftest_wait_timeout()
    assert qsa.device_status() == 4
    assert qsa.device_status() == 0          # read clears it
    wl = synth.make_workload(3, cells=700, rows=20)
    wl.top_k = 64
    cache, q, iq, iw = dev_inputs(qsa, wl)
    out = qsa.prefill_chunk(cache, wl.pos0, q, iq, iw, 64, wl.scale)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all() and qsa.device_status() == 0
