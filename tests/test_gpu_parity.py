"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle on the same
seeded inputs.  Sizes span several 128-key indexer tiles, several 64-key attention tiles and
ragged tails; full-size workloads are checked on seeded samples of rows."""
import math

import numpy as np
import pytest
import torch

import oracle
from dsa_workloads import FULL, TINY, make_config, make_decode, make_prefill, sample_rows
from tests.parity import (check_attention, check_scores, check_topk_exact, check_topk_layout,
                          n_valid_of, to_np, topk_overlap)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_04_b200 as m
    return m


def _ld(n):
    return (n + 3) // 4 * 4


def run_indexer(dsa, wl, rows_begin=0, rows_count=None):
    pb = dsa.problem_of(wl)
    T = wl.total_rows
    rows_count = T - rows_begin if rows_count is None else rows_count
    ld = _ld(wl.max_seqlen)
    scores = torch.full((rows_count, ld), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = dsa.dsa_indexer_scores(pb, wl.q_idx, wl.q_scale, wl.w, wl.k_idx, wl.k_scale,
                                rows_begin, rows_count, scores, ld, status)
    assert st == 0, dsa.status_string(st)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return scores


def run_topk(dsa, wl, scores, rows_begin=0, rows_count=None):
    pb = dsa.problem_of(wl)
    rows_count = scores.shape[0] if rows_count is None else rows_count
    idx = torch.empty(rows_count, wl.dims["topk"], dtype=torch.int32, device="cuda")
    st = dsa.dsa_topk(pb, scores, scores.shape[1], rows_begin, rows_count, idx)
    assert st == 0, dsa.status_string(st)
    torch.cuda.synchronize()
    return idx


def run_mla(dsa, wl, idx, rows_begin=0, rows_count=None):
    pb = dsa.problem_of(wl)
    T = wl.total_rows
    rows_count = idx.shape[0] if rows_count is None else rows_count
    d = wl.dims
    out = torch.full((T, d["h"], d["d_v"]), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((T, d["h"]), float("nan"), device="cuda")
    wsb = dsa.dsa_sparse_mla_workspace_size(pb, rows_count)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = dsa.dsa_sparse_mla_fwd(pb, wl.q, wl.kv, idx, rows_begin, rows_count, out, lse, ws, wsb,
                                status)
    assert st == 0, dsa.status_string(st)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out, lse


# ------------------------------------------------------------------------------- indexer

def _indexer_case(dsa, wl, rows):
    scores = run_indexer(dsa, wl)
    ref = oracle.indexer_rows(wl, rows)
    sc = to_np(scores)
    for r in rows:
        n = len(ref[r])
        check_scores(sc[r, :n], ref[r], f"row {r}")
    return scores


def test_indexer_tiny_prefill_all_rows(dsa):
    wl = make_config(1, device="cuda")
    _indexer_case(dsa, wl, list(range(wl.total_rows)))


def test_indexer_full_dims_varlen_prefill(dsa):
    wl = make_prefill(11, [130, 7, 600, 1, 515], FULL, needles=8, device="cuda")
    _indexer_case(dsa, wl, list(range(wl.total_rows)))


def test_indexer_decode_contiguous(dsa):
    wl = make_decode(12, 3, [5000, 130, 64], FULL, boost=0.01, paged=False, device="cuda")
    _indexer_case(dsa, wl, [0, 1, 2])


def test_indexer_decode_paged_ragged(dsa):
    wl = make_decode(13, 4, [3000, 64, 1, 200], FULL, boost=0.01, paged=True, device="cuda",
                     total_blocks=200)
    _indexer_case(dsa, wl, [0, 1, 2, 3])


def test_indexer_decode_paged_interleaved_scales(dsa):
    """The paged indexer cache with each block's scales after its key rows: scores equal,
    bit for bit, those of the same keys in separate arrays, and the oracle's."""
    lens = [3000, 64, 1, 200, 131]
    a = make_decode(17, 5, lens, FULL, boost=0.01, paged=True, device="cuda")
    b = make_decode(17, 5, lens, FULL, boost=0.01, paged=True, device="cuda",
                    scale_layout="interleaved")
    sa = run_indexer(dsa, a)
    sb = run_indexer(dsa, b)
    for r, n in enumerate(lens):
        assert torch.equal(sa[r, :n], sb[r, :n]), r
    ref = oracle.indexer_rows(b, list(range(5)))
    sc = to_np(sb)
    for r in range(5):
        check_scores(sc[r, :len(ref[r])], ref[r], f"row {r}")


def test_indexer_bad_block_reported(dsa):
    """A block-table entry that is negative or past the cache is skipped and reported as
    DSA_DEVICE_BAD_INDEX; the other sequences' scores are unaffected."""
    wl = make_decode(16, 3, [700, 300, 130], FULL, boost=0.01, paged=True, device="cuda",
                     total_blocks=40)
    good = oracle.indexer_rows(wl, [1, 2])
    wl.block_table[0, 3] = -1
    wl.block_table[0, 5] = 40          # one past the last physical block
    pb = dsa.problem_of(wl)
    ld = _ld(wl.max_seqlen)
    scores = torch.full((3, ld), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert dsa.dsa_indexer_scores(pb, wl.q_idx, wl.q_scale, wl.w, wl.k_idx, wl.k_scale, 0, 3,
                                  scores, ld, status) == 0
    torch.cuda.synchronize()
    assert int(status.item()) & dsa.DSA_DEVICE_BAD_INDEX
    sc = to_np(scores)
    for r in (1, 2):
        check_scores(sc[r, :len(good[r])], good[r], f"row {r}")


def test_indexer_row_subrange(dsa):
    wl = make_prefill(14, [300, 400], FULL, needles=8, device="cuda")
    scores = run_indexer(dsa, wl, rows_begin=250, rows_count=200)
    ref = oracle.indexer_rows(wl, list(range(250, 450)))
    sc = to_np(scores)
    for i, r in enumerate(range(250, 450)):
        check_scores(sc[i, :len(ref[r])], ref[r], f"row {r}")


# ------------------------------------------------------------------------------- top-k

@pytest.mark.parametrize("k", [64, 2048])
def test_topk_exact_synthetic(dsa, k):
    """Seeded score rows: Gaussian, heavy ties (small integers), all-equal, and lengths around k."""
    g = torch.Generator(device="cuda").manual_seed(5 + k)
    lens = [1, k - 1, k, k + 1, 3 * k + 17, 40000]
    wl_lens = lens
    T = len(lens)
    ld = _ld(max(lens))
    kinds = []
    rows = []
    for i, n in enumerate(lens):
        kind = i % 3
        if kind == 0:
            r = torch.randn(n, generator=g, device="cuda").abs()
        elif kind == 1:
            r = torch.randint(0, 5, (n,), generator=g, device="cuda").float()
        else:
            r = torch.zeros(n, device="cuda")
        rows.append(r)
        kinds.append(kind)
    scores = torch.zeros(T, ld, device="cuda")
    for i, r in enumerate(rows):
        scores[i, :len(r)] = r
    # decode geometry: row i has lens[i] keys
    pb = dsa.make_problem(mode="decode", h_idx=64, d_idx=128, h=128, d_qk=576, d_v=512, topk=k,
                          softmax_scale=1.0, num_kv_rows=T * max(wl_lens), seqlens=wl_lens,
                          seq_lens=torch.tensor(wl_lens, dtype=torch.int32, device="cuda"))
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    assert dsa.dsa_topk(pb, scores, ld, 0, T, idx) == 0
    torch.cuda.synchronize()
    sc, ix = to_np(scores), to_np(idx)
    for i, n in enumerate(lens):
        check_topk_exact(ix[i], sc[i, :n], k, f"row {i} n={n} kind={kinds[i]}")


def test_topk_cluster_paths(dsa):
    """Rows long enough to split over a cluster of CTAs: a resolvable first-digit bin (its keys
    gathered into one CTA), a crowded bin (every key in one bin: the digits are resolved by the
    whole cluster), ties across slice boundaries, ragged lengths, signed scores."""
    k = 2048
    g = torch.Generator(device="cuda").manual_seed(77)
    rows = [
        torch.randn(131072, generator=g, device="cuda").abs(),
        torch.randn(100003, generator=g, device="cuda"),
        1.0 + 0.25 * torch.rand(60000, generator=g, device="cuda"),
        torch.randint(0, 31, (50001,), generator=g, device="cuda").float(),
        1.0 + torch.randint(0, 4096, (70002,), generator=g, device="cuda").float() / 16384.0,
        torch.randn(16385, generator=g, device="cuda") * 1e-30,
        torch.full((32768,), 2.5, device="cuda"),
    ]
    lens = [len(r) for r in rows]
    ld = _ld(max(lens))
    scores = torch.zeros(len(rows), ld, device="cuda")
    for i, r in enumerate(rows):
        scores[i, :len(r)] = r
    pb = dsa.make_problem(mode="decode", h_idx=64, d_idx=128, h=128, d_qk=576, d_v=512, topk=k,
                          softmax_scale=1.0, num_kv_rows=len(rows) * max(lens), seqlens=lens,
                          seq_lens=torch.tensor(lens, dtype=torch.int32, device="cuda"))
    idx = torch.empty(len(rows), k, dtype=torch.int32, device="cuda")
    assert dsa.dsa_topk(pb, scores, ld, 0, len(rows), idx) == 0
    torch.cuda.synchronize()
    sc, ix = to_np(scores), to_np(idx)
    for i, n in enumerate(lens):
        check_topk_exact(ix[i], sc[i, :n], k, f"row {i} n={n}")


def test_topk_negative_and_signed_zero(dsa):
    k = 64
    g = torch.Generator(device="cuda").manual_seed(9)
    n = 1000
    r = torch.randn(n, generator=g, device="cuda")
    r[::7] = 0.0
    r[3::7] = -0.0
    scores = torch.zeros(1, _ld(n), device="cuda")
    scores[0, :n] = r
    pb = dsa.make_problem(mode="decode", h_idx=64, d_idx=128, h=128, d_qk=576, d_v=512, topk=k,
                          softmax_scale=1.0, num_kv_rows=n, seqlens=[n],
                          seq_lens=torch.tensor([n], dtype=torch.int32, device="cuda"))
    idx = torch.empty(1, k, dtype=torch.int32, device="cuda")
    assert dsa.dsa_topk(pb, scores, scores.shape[1], 0, 1, idx) == 0
    torch.cuda.synchronize()
    check_topk_exact(to_np(idx)[0], to_np(scores)[0, :n], k)


def test_topk_prefill_rows_on_indexer_scores(dsa):
    wl = make_prefill(15, [3000, 100], FULL, needles=8, device="cuda")
    scores = run_indexer(dsa, wl)
    idx = run_topk(dsa, wl, scores)
    sc, ix = to_np(scores), to_np(idx)
    rows = [0, 5, 2046, 2047, 2048, 2049, 2999, 3000, 3099]
    ref = oracle.indexer_rows(wl, rows)
    for r in rows:
        n = n_valid_of(wl, r)
        check_topk_exact(ix[r], sc[r, :n], 2048, f"row {r}")
    frac, viol = topk_overlap([ix[r] for r in rows], [ref[r] for r in rows], 2048)
    assert frac >= 0.999 and not viol, (frac, viol[:5])


# ------------------------------------------------------------------------------- sparse MLA

def _random_idx(wl, rows, k, g, holes=True):
    idx = torch.full((len(rows), k), -1, dtype=torch.int32)
    for i, r in enumerate(rows):
        n = n_valid_of(wl, r)
        m = min(n, k)
        sel = torch.randperm(n, generator=g)[:m].to(torch.int32)
        idx[i, :m] = sel
        if holes and m > 100:
            idx[i, 64:128] = -1          # a fully invalid tile
            idx[i, 7] = -1               # a hole inside a tile
    return idx


@pytest.mark.parametrize("shape", ["tiny", "full"])
def test_sparse_mla_prefill_synthetic_idx(dsa, shape):
    dims = TINY if shape == "tiny" else FULL
    wl = make_prefill(16, [700, 90], dims, needles=0, device="cuda")
    rows = list(range(wl.total_rows))
    g = torch.Generator().manual_seed(3)
    idx = _random_idx(wl, rows, dims["topk"], g)
    out, lse = run_mla(dsa, wl, idx.cuda())
    sample = rows[::7] + [699, 700, 789]
    ro, rl = oracle.sparse_mla_rows(wl, sample, idx[sample].numpy())
    o, l = to_np(out), to_np(lse)
    for i, r in enumerate(sample):
        check_attention(o[r], l[r], ro[i], rl[i], dims["h"], f"row {r}")


def test_sparse_mla_decode_split_kv(dsa):
    """Few rows: the kernel splits each row's tiles over several clusters and merges by LSE."""
    wl = make_decode(17, 2, [9000, 2500], FULL, boost=0.0, paged=True, device="cuda")
    g = torch.Generator().manual_seed(4)
    idx = _random_idx(wl, [0, 1], 2048, g)
    assert dsa.dsa_sparse_mla_workspace_size(dsa.problem_of(wl), 2) > 0
    out, lse = run_mla(dsa, wl, idx.cuda())
    ro, rl = oracle.sparse_mla_rows(wl, [0, 1], idx.numpy())
    for i in range(2):
        check_attention(to_np(out)[i], to_np(lse)[i], ro[i], rl[i], 128, f"row {i}")


def test_sparse_mla_large_logits_rescale(dsa):
    """Queries scaled so logits span far more than 2^8 within a row: exercises the lazy rescale."""
    wl = make_prefill(18, [600], FULL, needles=0, device="cuda")
    wl.q = (wl.q.float() * 6.0).to(torch.bfloat16)
    rows = [599, 300, 64]
    g = torch.Generator().manual_seed(6)
    idx = _random_idx(wl, rows, 2048, g, holes=False)
    # run rows one by one with row_begin = r so the idx row maps to row r
    for r, irow in zip(rows, idx):
        full_idx = irow.view(1, -1).cuda()
        out, lse = run_mla(dsa, wl, full_idx, rows_begin=r, rows_count=1)
        ro, rl = oracle.sparse_mla_rows(wl, [r], irow.view(1, -1).numpy())
        check_attention(to_np(out)[r], to_np(lse)[r], ro[0], rl[0], 128, f"row {r}")


def test_sparse_mla_bad_index_reported(dsa):
    wl = make_prefill(19, [300], FULL, needles=0, device="cuda")
    idx = torch.full((1, 2048), -1, dtype=torch.int32)
    idx[0, :10] = torch.arange(10)
    idx[0, 10] = 5000                      # beyond the row's position
    pb = dsa.problem_of(wl)
    out = torch.empty(300, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(300, 128, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert dsa.dsa_sparse_mla_fwd(pb, wl.q, wl.kv, idx.cuda(), 299, 1, out, lse, None, 0,
                                  status) == 0
    st, raw = dsa.dsa_read_device_status(status)
    assert st == dsa.DSA_ERR_BAD_INDEX and raw & dsa.DSA_DEVICE_BAD_INDEX
    ro, rl = oracle.sparse_mla_rows(wl, [299], np.where(idx.numpy() == 5000, -1, idx.numpy()))
    check_attention(to_np(out)[299], to_np(lse)[299], ro[0], rl[0], 128)


# ------------------------------------------------------------------------------- whole path

def _forward(dsa, wl):
    f = dsa.Forward(wl)
    st = f()
    assert st == 0, dsa.status_string(st)
    torch.cuda.synchronize()
    assert int(f.status.item()) == 0
    return f


def _check_forward(wl, f, rows, overlap_min=0.999):
    sc_ref, idx_ref, o_ref, l_ref = None, None, None, None
    ref_scores = oracle.indexer_rows(wl, rows)
    gidx = to_np(f.idx)[rows]
    for i, r in enumerate(rows):
        check_topk_layout(gidx[i], n_valid_of(wl, r), wl.dims["topk"], f"row {r}")
    frac, viol = topk_overlap(list(gidx), [ref_scores[r] for r in rows], wl.dims["topk"])
    assert frac >= overlap_min and not viol, (frac, viol[:5])
    ro, rl = oracle.sparse_mla_rows(wl, rows, gidx)
    o, l = to_np(f.out), to_np(f.lse)
    for i, r in enumerate(rows):
        check_attention(o[r], l[r], ro[i], rl[i], wl.dims["h"], f"row {r}")


def test_forward_tiny_prefill_all_rows(dsa):
    wl = make_config(1, device="cuda")
    f = _forward(dsa, wl)
    _check_forward(wl, f, list(range(wl.total_rows)))


def test_forward_small_decode_full_dims(dsa):
    wl = make_decode(21, 5, [7000, 2048, 2049, 100, 1], FULL, boost=0.01, paged=True,
                     device="cuda")
    f = _forward(dsa, wl)
    _check_forward(wl, f, [0, 1, 2, 3, 4])


def test_forward_small_prefill_full_dims(dsa):
    wl = make_prefill(22, [2500, 300], FULL, needles=8, device="cuda")
    f = _forward(dsa, wl)
    rows = [0, 1, 63, 2046, 2047, 2048, 2100, 2499, 2500, 2799]
    _check_forward(wl, f, rows)


# ------------------------------------------------------ per-head query scales of the indexer

def per_head_q_scale(wl, seed):
    """The workload with a different fp32 scale for every (query row, indexer head): the
    generator draws one scale per token (copied over the heads); here each head's scale is
    multiplied by its own seeded power-of-two-spread factor in [1/8, 8).  Both sides read the
    same modified array."""
    g = torch.Generator(device=wl.q_scale.device).manual_seed(seed)
    f = torch.exp2(torch.rand(wl.q_scale.shape, generator=g, device=wl.q_scale.device) * 6 - 3)
    wl.q_scale = (wl.q_scale * f).contiguous()
    assert (wl.q_scale[:, 0] != wl.q_scale[:, 1]).any()
    return wl


def test_indexer_per_head_q_scale(dsa):
    _indexer_case(dsa, per_head_q_scale(make_config(1, device="cuda"), 5), list(range(1024)))
    wl = make_prefill(11, [130, 7, 600, 1, 515], FULL, needles=8, device="cuda")
    _indexer_case(dsa, per_head_q_scale(wl, 6), list(range(wl.total_rows)))
    for lay in ("separate", "interleaved"):
        wl = make_decode(17, 5, [3000, 64, 1, 200, 131], FULL, boost=0.01, paged=True,
                         device="cuda", scale_layout=lay)
        _indexer_case(dsa, per_head_q_scale(wl, 7), list(range(5)))


def test_forward_per_head_q_scale(dsa):
    wl = per_head_q_scale(make_decode(21, 5, [7000, 2048, 2049, 100, 1], FULL, boost=0.01,
                                      paged=True, device="cuda"), 8)
    _check_forward(wl, _forward(dsa, wl), [0, 1, 2, 3, 4])
    wl = per_head_q_scale(make_prefill(22, [2500, 300], FULL, needles=8, device="cuda"), 9)
    _check_forward(wl, _forward(dsa, wl), [0, 1, 63, 2046, 2047, 2048, 2100, 2499, 2500, 2799])


# --------------------------------------------------------------- dense (short-row) attention

def test_sparse_mla_dense_equals_sparse_with_all_keys(dsa):
    """Without an index array the attention takes every prior key; for rows with at most topk
    prior keys that is exactly the top-k's selection, so the result is bit-identical to the
    sparse call on the top-k's indices, and matches the oracle."""
    wl = make_prefill(41, [2048, 700], FULL, needles=8, device="cuda")
    T = wl.total_rows
    scores = run_indexer(dsa, wl)
    idx = run_topk(dsa, wl, scores)
    o_s, l_s = run_mla(dsa, wl, idx)
    pb = dsa.problem_of(wl)
    d = wl.dims
    o_d = torch.full((T, d["h"], d["d_v"]), float("nan"), dtype=torch.bfloat16, device="cuda")
    l_d = torch.full((T, d["h"]), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert dsa.dsa_sparse_mla_fwd(pb, wl.q, wl.kv, None, 0, T, o_d, l_d, None, 0, status) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(o_d.view(torch.int16), o_s.view(torch.int16))
    assert torch.equal(l_d, l_s)
    rows = list(range(0, T, 37)) + [2047, 2048, T - 1]
    dense_idx = np.full((len(rows), d["topk"]), -1, dtype=np.int32)
    for i, r in enumerate(rows):
        n = n_valid_of(wl, r)
        dense_idx[i, :n] = np.arange(n)
    ro, rl = oracle.sparse_mla_rows(wl, rows, dense_idx)
    o, l = to_np(o_d), to_np(l_d)
    for i, r in enumerate(rows):
        check_attention(o[r], l[r], ro[i], rl[i], d["h"], f"row {r}")


def test_forward_without_indices_dense_first_rows(dsa):
    """dsa_forward with no index output: the first topk rows of each sequence run dense (no
    indexer, no top-k) and match the oracle (whose selection is every key there); the later
    rows take the sparse path and equal, bit for bit, a run that keeps the indices."""
    wl = make_config(1, device="cuda")                 # L = 1024, topk = 64
    f = dsa.Forward(wl, keep_idx=False)
    assert f() == 0
    g = dsa.Forward(wl, keep_idx=True)
    assert g() == 0
    torch.cuda.synchronize()
    assert int(f.status.item()) == 0 and int(g.status.item()) == 0
    rows = list(range(0, 64))
    _, _, o_ref, l_ref = oracle.forward_rows(wl, rows)
    o, l = to_np(f.out), to_np(f.lse)
    for i, r in enumerate(rows):
        check_attention(o[r], l[r], o_ref[i], l_ref[i], wl.dims["h"], f"row {r}")
    assert torch.equal(f.out[64:].view(torch.int16), g.out[64:].view(torch.int16))
    assert torch.equal(f.lse[64:], g.lse[64:])


def test_forward_short_decode_is_dense(dsa):
    """A decode batch whose contexts all fit in topk keeps every key: dsa_forward skips the
    indexer and the top-k and matches the oracle's whole pipeline."""
    wl = make_decode(42, 4, [2048, 1, 900, 64], FULL, boost=0.01, paged=True, device="cuda")
    f = dsa.Forward(wl, keep_idx=False)
    assert f() == 0
    torch.cuda.synchronize()
    assert int(f.status.item()) == 0
    rows = [0, 1, 2, 3]
    _, idx_ref, o_ref, l_ref = oracle.forward_rows(wl, rows)
    o, l = to_np(f.out), to_np(f.lse)
    for i, r in enumerate(rows):
        check_attention(o[r], l[r], o_ref[i], l_ref[i], wl.dims["h"], f"row {r}")
