"""The fused indexer + top-k (dsa_indexer_topk) on the GPU.

The indexer counts each row's first radix digit as it writes the scores and the selection starts
from those counts.  Checks, on the same seeded inputs:
  - the selection is exactly the oracle's selector applied to the GPU's own scores (the scores of
    dsa_indexer_scores, which the fused call computes with the same kernel), bit for bit;
  - it is identical to the unfused pair dsa_indexer_scores + dsa_topk;
  - against the oracle's own scores: >= 99.9 % overlap, every miss within the score tolerance;
  - degenerate rows: all scores equal (w = 0: every score is +0, so the first topk keys win),
    negative scores (w < 0), rows shorter than topk, row sub-ranges, paged caches with the scales
    inside the pages, and the 4 x 32 indexer (no fused histogram: the selection builds its own);
  - the whole path (dsa_forward) on a chunked prefill, whose chunks reuse the histograms.
"""
import numpy as np
import pytest
import torch

import oracle
from dsa_workloads import FULL, make_config, make_decode, make_prefill
from tests.parity import check_topk_exact, check_topk_layout, n_valid_of, to_np, topk_overlap

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_04_b200 as m
    return m


def _fused(dsa, wl, rb, n, with_sel=False):
    pb = dsa.problem_of(wl)
    ws_bytes = dsa.dsa_indexer_topk_workspace_size(pb, n)
    assert ws_bytes > 0
    ws = torch.full((ws_bytes,), 0xA5, dtype=torch.uint8, device="cuda")   # junk on entry
    idx = torch.full((n, wl.dims["topk"]), -7, dtype=torch.int32, device="cuda")
    sel = (torch.full((n, wl.dims["topk"]), float("nan"), device="cuda") if with_sel
           else None)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = dsa.dsa_indexer_topk(pb, wl.q_idx, wl.q_scale, wl.w, wl.k_idx, wl.k_scale, rb, n, idx,
                              ws, ws_bytes, status, sel_out=sel)
    assert st == dsa.DSA_OK, dsa.status_string(st)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return (to_np(idx), to_np(sel)) if with_sel else to_np(idx)


def _check_sel(idx, sel, sc):
    """sel[t][e] = the slab's score of key idx[t][e], bit for bit; 0 where idx is -1."""
    for i in range(idx.shape[0]):
        ok = idx[i] >= 0
        assert np.array_equal(sel[i, ok].view(np.uint32), sc[i, idx[i, ok]].view(np.uint32)), i
        assert not sel[i, ~ok].any(), i


def _unfused(dsa, wl, rb, n):
    pb = dsa.problem_of(wl)
    ld = (wl.max_seqlen + 3) // 4 * 4
    sc = torch.full((n, ld), float("nan"), device="cuda")
    assert dsa.dsa_indexer_scores(pb, wl.q_idx, wl.q_scale, wl.w, wl.k_idx, wl.k_scale, rb, n, sc,
                                  ld) == dsa.DSA_OK
    idx = torch.empty(n, wl.dims["topk"], dtype=torch.int32, device="cuda")
    assert dsa.dsa_topk(pb, sc, ld, rb, n, idx) == dsa.DSA_OK
    torch.cuda.synchronize()
    return to_np(sc), to_np(idx)


def _check(dsa, wl, rb, n, oracle_rows=None, overlap=True):
    got, sel = _fused(dsa, wl, rb, n, with_sel=True)
    sc, ref_idx = _unfused(dsa, wl, rb, n)
    k = wl.dims["topk"]
    assert np.array_equal(got, ref_idx)
    _check_sel(got, sel, sc)
    for i in range(n):
        nv = n_valid_of(wl, rb + i)
        check_topk_exact(got[i], sc[i, :nv], k, f"row {rb + i}")
    if overlap:
        rows = list(range(rb, rb + n)) if oracle_rows is None else oracle_rows
        ref = oracle.indexer_rows(wl, rows)
        frac, viol = topk_overlap([got[r - rb] for r in rows], [ref[r] for r in rows], k)
        assert frac >= 0.999 and not viol, (frac, viol[:5])
    return got


def test_fused_decode_paged(dsa):
    for lay in ("separate", "interleaved"):
        wl = make_decode(61, 6, [131072, 9000, 2049, 2048, 700, 1], FULL, boost=0.005,
                         paged=True, device="cuda", scale_layout=lay)
        _check(dsa, wl, 0, 6)


def test_fused_decode_contiguous_subrange(dsa):
    wl = make_decode(62, 5, [5000, 30000, 4100, 100, 65536], FULL, boost=0.01, paged=False,
                     device="cuda")
    _check(dsa, wl, 1, 3)


def test_fused_prefill_varlen(dsa):
    wl = make_prefill(63, [5000, 300, 2049, 7000], FULL, needles=8, device="cuda")
    T = wl.total_rows
    rows = [0, 2047, 2048, 2100, 4999, 5000, 5299, 5300 + 2048, 7348 + 10, T - 1]
    _check(dsa, wl, 0, T, oracle_rows=rows)


def test_fused_ties_and_negative_scores(dsa):
    """w = 0 makes every score of a row +0 (mass ties: the first topk keys are selected); w < 0
    makes them <= 0."""
    wl = make_decode(64, 4, [40000, 6000, 3000, 70000], FULL, boost=0.0, paged=True,
                     device="cuda")
    wl.w[0].zero_()
    wl.w[2] = -wl.w[2]
    got = _check(dsa, wl, 0, 4, overlap=False)
    assert np.array_equal(got[0], np.arange(2048, dtype=np.int32))
    wl = make_prefill(65, [6000], FULL, needles=8, device="cuda")
    wl.w[3000:3100].zero_()
    wl.w[4000:4100] = -wl.w[4000:4100]
    got = _check(dsa, wl, 2990, 1200, overlap=False)
    assert np.array_equal(got[3050 - 2990], np.arange(2048, dtype=np.int32))


def test_fused_small_indexer_shape(dsa):
    wl = make_config(1, device="cuda")
    _check(dsa, wl, 0, wl.total_rows, oracle_rows=list(range(0, 1024, 7)))


def test_forward_chunked_prefill_reuses_histograms(dsa):
    """A prefill long enough for several row chunks of the forward: every chunk's selection
    equals the fused call's on the same rows (the forward keeps its indices)."""
    wl = make_prefill(66, [70000], FULL, needles=8, device="cuda")
    pb = dsa.problem_of(wl)
    f = dsa.Forward(wl, keep_sel=True)
    assert f() == dsa.DSA_OK
    torch.cuda.synchronize()
    assert int(f.status.item()) == 0
    gidx, gsel = to_np(f.idx), to_np(f.sel)
    for rb, n in ((0, 100), (2048, 300), (40000, 200), (69800, 200)):
        got, sel = _fused(dsa, wl, rb, n, with_sel=True)
        assert np.array_equal(gidx[rb:rb + n], got), rb
        assert np.array_equal(gsel[rb:rb + n].view(np.uint32), sel.view(np.uint32)), rb
    rows = [2048, 30000, 69999]
    ref = oracle.indexer_rows(wl, rows)
    for r in rows:
        check_topk_layout(gidx[r], n_valid_of(wl, r), 2048, f"row {r}")
    frac, viol = topk_overlap([gidx[r] for r in rows], [ref[r] for r in rows], 2048)
    assert frac >= 0.999 and not viol, (frac, viol[:5])


def test_staged_calls_with_histograms(dsa):
    """dsa_indexer_scores counting into caller-owned histograms, then dsa_topk starting from
    them: the same selection as the fused call, and the histograms are zero again afterwards
    (ready for the next rows).  The counts themselves are checked against the scores."""
    wl = make_decode(67, 5, [131072, 30000, 2049, 500, 77777], FULL, boost=0.005, paged=True,
                     device="cuda", scale_layout="interleaved")
    pb = dsa.problem_of(wl)
    n = 5
    ld = (wl.max_seqlen + 3) // 4 * 4
    sc = torch.empty(n, ld, device="cuda")
    hist = torch.zeros(n, dsa.TOPK_HIST_BINS, dtype=torch.int32, device="cuda")
    assert dsa.dsa_indexer_scores(pb, wl.q_idx, wl.q_scale, wl.w, wl.k_idx, wl.k_scale, 0, n, sc,
                                  ld, hist=hist) == dsa.DSA_OK
    torch.cuda.synchronize()
    s_np, h_np = to_np(sc), to_np(hist).astype(np.int64)
    for i, L in enumerate(wl.seqlens):
        bits = s_np[i, :L].view(np.uint32).astype(np.uint64)
        bits[(bits & 0x7FFFFFFF) == 0] = 0                       # -0 counts as +0
        key = np.where(bits & 0x80000000, ~bits & 0xFFFFFFFF, bits | 0x80000000)
        ref_h = np.bincount((key >> 21).astype(np.int64), minlength=2048)
        assert np.array_equal(h_np[i], ref_h), i
    idx = torch.empty(n, 2048, dtype=torch.int32, device="cuda")
    sel = torch.full((n, 2048), float("nan"), device="cuda")
    assert dsa.dsa_topk(pb, sc, ld, 0, n, idx, hist=hist, sel_out=sel) == dsa.DSA_OK
    torch.cuda.synchronize()
    assert not hist.any()
    _check_sel(to_np(idx), to_np(sel), s_np)
    assert np.array_equal(to_np(idx), _fused(dsa, wl, 0, n))
    for i, L in enumerate(wl.seqlens):
        check_topk_exact(to_np(idx)[i], s_np[i, :L], 2048, f"row {i}")
