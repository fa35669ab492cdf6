"""The selection call that needs no workspace (qsa_topk_static) against the
workspace version (qsa_topk) and the CPU oracle, through the C ABI.

It serves callers that cannot allocate device memory at the point of the call
(inside a CUDA graph capture, in serving loops that must avoid allocator calls
and their implicit synchronisation, or under a memory budget owned by another
allocator).  Two calls in a row on different scores must each match qsa_topk
exactly, and the oracle's selection on the same fp32 scores (widened exactly to
float64, so both decide on the same values) -- the second call also shows the
shared scratch buffer is cleared between calls.  The file is named to be collected last, and passes both alone in a
fresh process (where its first call looks up the buffer) and after the others.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def _scores(seed, rows, cells, ties):
    st = synth.Stream(seed, "no_alloc")
    s = st.normal(rows * cells).reshape(rows, cells)
    if ties:
        s = np.round(s * 3) / 3
    return torch.from_numpy(s.astype(np.float32)).to("cuda:0")


def _static_topk(lib, scores, vis0, top_k):
    rows, ld = scores.shape
    ids = torch.full((rows, top_k), -7, dtype=torch.int32, device="cuda:0")
    rc = lib.qsa_topk_static(ctypes.c_void_p(scores.data_ptr()), ld, rows, vis0, top_k,
                             ctypes.c_void_p(ids.data_ptr()),
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, lib.qsa_last_error().decode()
    return ids


def test_static_topk_matches_workspace_topk(gpu):
    qsa = gpu
    lib = qsa.load()
    cases = [(_scores(1, 8, 65536, False), 65529, 2048),   # 8 decode rows at 64K cells
             (_scores(2, 3, 20000, True), 19998, 1500)]    # fewer rows, many tied scores
    for scores, vis0, top_k in cases:                      # two calls in a row
        got = _static_topk(lib, scores, vis0, top_k)
        want = qsa.topk(scores, vis0, top_k)
        torch.cuda.synchronize()
        assert torch.equal(got, want)
        host, ids = scores.cpu().numpy(), got.cpu().numpy()
        for r in range(host.shape[0]):
            ref = oracle.topk(host[r, :vis0 + r].astype(np.float64), top_k)
            assert np.array_equal(ids[r], ref), r


def test_static_topk_rejects_oversize(gpu):
    qsa = gpu
    lib = qsa.load()
    scores = _scores(3, 9, 4096, False)
    ids = torch.empty(9, 64, dtype=torch.int32, device="cuda:0")
    before = qsa.launch_count()
    rc = lib.qsa_topk_static(ctypes.c_void_p(scores.data_ptr()), 4096, 9, 4000, 64,
                             ctypes.c_void_p(ids.data_ptr()), None)
    assert rc == 1 and "rows = 9" in lib.qsa_last_error().decode()
    rc = lib.qsa_topk_static(ctypes.c_void_p(scores.data_ptr()), 4096, 2, 4000, 2049,
                             ctypes.c_void_p(ids.data_ptr()), None)
    assert rc == 1 and "top_k = 2049" in lib.qsa_last_error().decode()
    assert qsa.launch_count() == before
