"""The indexer's training step on the GPU against the oracle: the KL target (the main attention's
head-summed distribution on the selected keys) and the KL loss with its gradients for w, q, k.

Every input the oracle sees comes from the seeded generators or from the oracle itself: the
selection is the oracle's own top-k, the LSE the oracle's attention, the target the oracle's.
The GPU gets the same values (the LSE and the target rounded to fp32).

Tolerances (derived from the arithmetic):
  target   |t_gpu - t_ref| <= 1e-4 t_ref + 1e-7: fp32 logits from exact bf16 products (relative
           error ~1e-6 at logits of order 1), one exp2 and a 128-head fp32 sum
  loss     |L_gpu - L_ref| <= 1e-3 |L_ref| + 1e-5: the fp32 indexer scores carry the indexer's
           1e-3 relative tolerance into the softmax
  grads    element by element, |g_gpu - g_ref| <= 2e-3 |g_ref| + 1e-4 M, with M = max|g_ref|
           over the whole gradient tensor (dw, dq, or every touched key of dk); and per row
           rel-L2 <= 2e-3 in the sparse stage.  The coefficient g_e = pi_e sum p - p_e of a key
           cancels to ~0 where the indexer already matches the target, so an element's own size
           is no scale for its error: an absolute score error eta moves g_e by up to 2 eta pi_e,
           a shift set by the row's probabilities, not by g_e.  A gradient row sums such terms
           over up to 2048 selected keys (the dense warm-up: every prior key) and can cancel as a
           whole (g sums to 0 over a row whose target sums to 1), so the floor is the tensor's
           scale, not the row's own.  The dense warm-up's rows sum every prior key: there the
           floor is 1e-3 of the tensor's scale, with the per-row rel-L2 bound beside it.
"""
import numpy as np
import pytest
import torch

import oracle
from dsa_workloads import FULL, make_config, make_decode, make_prefill
from tests.parity import to_np

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

T_REL, T_ABS = 1e-4, 1e-7
L_REL, L_ABS = 1e-3, 1e-5
G_REL_L2 = 2e-3
G_REL, G_FLOOR = 2e-3, 1e-4
DENSE_FLOOR = 1e-3


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_04_b200 as m
    return m


def _oracle_selection(wl, rows):
    """The oracle's own top-k of its own scores, and its attention LSE on that selection."""
    sc = oracle.indexer_rows(wl, rows)
    idx = oracle.topk_rows([sc[r] for r in rows], wl.dims["topk"])
    _, lse = oracle.sparse_mla_rows(wl, rows, idx)
    return sc, idx, lse


def _gpu_target(dsa, wl, rb, idx, lse_rows):
    n, k = idx.shape
    lse = torch.zeros(wl.total_rows, wl.dims["h"], device="cuda")
    lse[rb:rb + n] = torch.tensor(lse_rows, dtype=torch.float32, device="cuda")
    idx_d = torch.tensor(idx, device="cuda")
    tgt = torch.full((n, k), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = dsa.dsa_indexer_kl_target(dsa.problem_of(wl), wl.q, wl.kv, idx_d, lse, rb, n, tgt,
                                   status, 0)
    assert st == dsa.DSA_OK, dsa.status_string(st)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return to_np(tgt)


def _check_target(got, ref, idx):
    assert not np.isnan(got).any()
    assert (got[idx < 0] == 0).all()
    err = np.abs(got - ref)
    bad = np.argwhere(err > T_REL * np.abs(ref) + T_ABS)
    assert len(bad) == 0, (bad[:5], got[tuple(bad[0])], ref[tuple(bad[0])])


def _rows_target(dsa, wl, rb, n):
    rows = list(range(rb, rb + n))
    _, idx, lse = _oracle_selection(wl, rows)
    got = _gpu_target(dsa, wl, rb, idx, lse)
    _check_target(got, oracle.kl_target_rows(wl, rows, idx), idx)
    return rows, idx, got


def test_kl_target_tiny_prefill(dsa):
    wl = make_config(1, device="cuda")
    _rows_target(dsa, wl, 0, 40)          # rows with fewer keys than k: holes in the selection
    _rows_target(dsa, wl, 980, 44)


def test_kl_target_full_dims_prefill_and_decode(dsa):
    wl = make_prefill(22, [2500, 300], FULL, needles=8, device="cuda")
    _rows_target(dsa, wl, 2040, 16)       # around pos + 1 = topk
    _rows_target(dsa, wl, 2490, 20)       # the end of one sequence and the start of the next
    wl = make_decode(21, 5, [7000, 2048, 2049, 100, 1], FULL, boost=0.01, paged=True,
                     device="cuda")       # split across CTAs (few rows), paged keys
    _rows_target(dsa, wl, 0, 5)


def test_kl_target_dense_without_indices(dsa):
    """No index array: every prior key, in position order (rows with at most k prior keys)."""
    wl = make_config(1, device="cuda")
    rows = list(range(0, 64))
    idx = np.array([list(range(t + 1)) + [-1] * (63 - t) for t in rows], np.int32)
    _, lse = oracle.sparse_mla_rows(wl, rows, idx)
    lse_d = torch.zeros(wl.total_rows, wl.dims["h"], device="cuda")
    lse_d[:64] = torch.tensor(lse, dtype=torch.float32, device="cuda")
    tgt = torch.full((64, 64), float("nan"), device="cuda")
    assert dsa.dsa_indexer_kl_target(dsa.problem_of(wl), wl.q, wl.kv, None, lse_d, 0, 64, tgt,
                                     None, 0) == dsa.DSA_OK
    torch.cuda.synchronize()
    _check_target(to_np(tgt), oracle.kl_target_rows(wl, rows, idx), idx)


def _gpu_backward(dsa, wl, rb, idx, target, sel=None):
    n, k = idx.shape
    d = wl.dims
    dev = "cuda"
    idx_d = torch.tensor(idx, device=dev)
    sel_d = None if sel is None else torch.tensor(sel, dtype=torch.float32, device=dev)
    tgt = torch.tensor(target, dtype=torch.float32, device=dev)
    loss = torch.full((n,), float("nan"), device=dev)
    dw = torch.full((n, d["h_idx"]), float("nan"), device=dev)
    dq = torch.full((n, d["h_idx"], d["d_idx"]), float("nan"), device=dev)
    dk = torch.zeros(wl.kv.shape[0], d["d_idx"], device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    st = dsa.dsa_indexer_kl_backward(dsa.problem_of(wl), wl.q_idx, wl.q_scale, wl.w, wl.k_idx,
                                     wl.k_scale, idx_d, tgt, rb, n, loss, dw, dq, dk, status, 0,
                                     sel=sel_d)
    assert st == dsa.DSA_OK, dsa.status_string(st)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return to_np(loss), to_np(dw), to_np(dq), to_np(dk)


def _rel_l2(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / nb if nb > 0 else np.linalg.norm(a)


def _check_elementwise(got, ref, what, per_row=False, floor=G_FLOOR):
    """|got - ref| <= G_REL |ref| + floor M, element by element; M = max|ref| of the element's
    row (first axis) or, with per_row False, of the whole tensor."""
    got = np.asarray(got, np.float64).reshape(len(ref), -1)
    ref = np.asarray(ref, np.float64).reshape(len(ref), -1)
    scale = (np.abs(ref).max(axis=1, keepdims=True) if per_row
             else np.abs(ref).max(initial=0.0))
    tol = G_REL * np.abs(ref) + floor * scale
    err = np.abs(got - ref)
    bad = np.argwhere(err > tol)
    assert len(bad) == 0, (what, len(bad), bad[:3].tolist(),
                           float((err / np.maximum(tol, 1e-30)).max()))


def _check_backward(dsa, wl, rb, n, with_sel=False):
    """with_sel: the selected keys' scores are passed in (the oracle's, in fp32), as the forward's
    selection hands them over; the kernel then takes the softmax over them."""
    rows = list(range(rb, rb + n))
    sc, idx, _ = _oracle_selection(wl, rows)
    target = oracle.kl_target_rows(wl, rows, idx).astype(np.float32)
    ref = oracle.indexer_kl_rows(wl, rows, idx, target.astype(np.float64))
    sel = None
    if with_sel:
        sel = np.zeros(idx.shape, np.float32)
        for i, r in enumerate(rows):
            ok = idx[i] >= 0
            sel[i, ok] = sc[r][idx[i, ok]]
    loss, dw, dq, dk = _gpu_backward(dsa, wl, rb, idx, target, sel)
    np.testing.assert_allclose(loss, ref["loss"], rtol=L_REL, atol=L_ABS)
    for i in range(n):
        assert _rel_l2(dw[i], ref["dw"][i]) <= G_REL_L2, ("dw", rows[i])
        assert _rel_l2(dq[i], ref["dq"][i]) <= G_REL_L2, ("dq", rows[i])
    _check_elementwise(dw, ref["dw"], "dw")
    _check_elementwise(dq, ref["dq"], "dq")
    _check_elementwise(dk[ref["dk_rows"]], ref["dk"], "dk")
    assert _rel_l2(dk[ref["dk_rows"]], ref["dk"]) <= G_REL_L2
    untouched = np.setdiff1d(np.arange(dk.shape[0]), ref["dk_rows"])
    assert not dk[untouched].any()


def test_kl_backward_tiny_prefill(dsa):
    wl = make_config(1, device="cuda")
    _check_backward(dsa, wl, 0, 40)
    _check_backward(dsa, wl, 980, 44)


def test_kl_backward_full_dims_prefill(dsa):
    wl = make_prefill(22, [2500, 300], FULL, needles=8, device="cuda")
    _check_backward(dsa, wl, 2040, 16)
    _check_backward(dsa, wl, 2490, 20)


def test_kl_backward_per_head_q_scale(dsa):
    """Every (row, indexer head) with its own query scale: the backward stages the scales per
    head, apart from w."""
    from tests.test_gpu_parity import per_head_q_scale
    wl = per_head_q_scale(make_prefill(22, [2500, 300], FULL, needles=8, device="cuda"), 10)
    _check_backward(dsa, wl, 2040, 16)
    wl = per_head_q_scale(make_config(1, device="cuda"), 11)
    _check_backward(dsa, wl, 980, 44)


def test_kl_backward_full_dims_paged_decode(dsa):
    wl = make_decode(21, 5, [7000, 2048, 2049, 100, 1], FULL, boost=0.01, paged=True,
                     device="cuda")
    _check_backward(dsa, wl, 0, 5)


def test_kl_backward_with_selected_scores(dsa):
    """The scores of the selected keys given (the forward's sel_out): pass 1 reads them instead
    of the keys; the same tolerances hold."""
    wl = make_config(1, device="cuda")
    _check_backward(dsa, wl, 980, 44, with_sel=True)
    wl = make_prefill(22, [2500, 300], FULL, needles=8, device="cuda")
    _check_backward(dsa, wl, 2040, 16, with_sel=True)
    _check_backward(dsa, wl, 2490, 20, with_sel=True)
    wl = make_decode(21, 5, [7000, 2048, 2049, 100, 1], FULL, boost=0.01, paged=True,
                     device="cuda")
    _check_backward(dsa, wl, 0, 5, with_sel=True)


def test_kl_backward_bad_index_reported(dsa):
    wl = make_config(1, device="cuda")
    rows = list(range(100, 104))
    _, idx, _ = _oracle_selection(wl, rows)
    target = oracle.kl_target_rows(wl, rows, idx)
    bad = idx.copy()
    bad[1, 3] = 5000                       # past the row's keys: skipped and reported
    ref_idx = bad.copy()
    ref_idx[1, 3] = -1
    ref = oracle.indexer_kl_rows(wl, rows, ref_idx, target)
    n, k = idx.shape
    loss = torch.zeros(n, device="cuda")
    dw = torch.zeros(n, 4, device="cuda")
    dq = torch.zeros(n, 4, 32, device="cuda")
    dk = torch.zeros(wl.kv.shape[0], 32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = dsa.dsa_indexer_kl_backward(dsa.problem_of(wl), wl.q_idx, wl.q_scale, wl.w, wl.k_idx,
                                     wl.k_scale, torch.tensor(bad, device="cuda"),
                                     torch.tensor(target, dtype=torch.float32, device="cuda"),
                                     100, n, loss, dw, dq, dk, status, 0)
    assert st == dsa.DSA_OK
    torch.cuda.synchronize()
    assert int(status.item()) & dsa.DSA_DEVICE_BAD_INDEX
    np.testing.assert_allclose(to_np(loss), ref["loss"], rtol=L_REL, atol=L_ABS)


# ------------------------------------------------------------------ dense warm-up stage

def _dense_idx(wl, rows):
    """Every prior key of each row, in position order, padded with -1 to the longest row."""
    from tests.parity import n_valid_of
    n = [n_valid_of(wl, r) for r in rows]
    idx = np.full((len(rows), max(n)), -1, np.int32)
    for i, m in enumerate(n):
        idx[i, :m] = np.arange(m)
    return idx


def _dense_case(dsa, wl, rb, n):
    """Dense attention (the LSE the warm-up target needs), the dense target and the dense KL
    backward of rows [rb, rb + n) against the oracle over every prior key."""
    from tests.parity import check_attention
    rows = list(range(rb, rb + n))
    idx = _dense_idx(wl, rows)
    ld = (idx.shape[1] + 63) // 64 * 64
    ld = max(ld, wl.dims["topk"])
    pb = dsa.problem_of(wl)
    d = wl.dims
    # 1. dense attention: out and LSE over every prior key
    o_ref, l_ref = oracle.sparse_mla_rows(wl, rows, idx)
    out = torch.full((wl.total_rows, d["h"], d["d_v"]), float("nan"), dtype=torch.bfloat16,
                     device="cuda")
    lse = torch.full((wl.total_rows, d["h"]), float("nan"), device="cuda")
    assert dsa.dsa_sparse_mla_fwd(pb, wl.q, wl.kv, None, rb, n, out, lse) == dsa.DSA_OK
    torch.cuda.synchronize()
    o, l = to_np(out), to_np(lse)
    for i, r in enumerate(rows):
        check_attention(o[r], l[r], o_ref[i], l_ref[i], d["h"], f"dense row {r}")
    # 2. the dense target from the oracle's LSE
    lse_d = torch.zeros(wl.total_rows, d["h"], device="cuda")
    lse_d[rb:rb + n] = torch.tensor(l_ref, dtype=torch.float32, device="cuda")
    tgt = torch.full((n, ld), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = dsa.dsa_indexer_kl_target_dense(pb, wl.q, wl.kv, lse_d, rb, n, tgt, ld, status)
    assert st == dsa.DSA_OK, dsa.status_string(st)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_t = oracle.kl_target_rows(wl, rows, idx)
    got_t = to_np(tgt)
    for i in range(n):
        m = int((idx[i] >= 0).sum())
        _check_target(got_t[i:i + 1, :m], ref_t[i:i + 1, :m], idx[i:i + 1, :m])
        assert np.allclose(ref_t[i, :m].sum(), 1.0)
    # 3. the dense KL backward on the oracle's target
    target = ref_t.astype(np.float32)
    ref = oracle.indexer_kl_rows(wl, rows, idx, target.astype(np.float64))
    t_pad = np.zeros((n, ld), np.float32)
    t_pad[:, :target.shape[1]] = target
    loss = torch.full((n,), float("nan"), device="cuda")
    dw = torch.full((n, d["h_idx"]), float("nan"), device="cuda")
    dq = torch.full((n, d["h_idx"], d["d_idx"]), float("nan"), device="cuda")
    dk = torch.zeros(wl.kv.shape[0], d["d_idx"], device="cuda")
    st = dsa.dsa_indexer_kl_backward_dense(pb, wl.q_idx, wl.q_scale, wl.w, wl.k_idx, wl.k_scale,
                                           torch.tensor(t_pad, device="cuda"), ld, rb, n, loss,
                                           dw, dq, dk, status)
    assert st == dsa.DSA_OK, dsa.status_string(st)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    loss, dw, dq, dk = to_np(loss), to_np(dw), to_np(dq), to_np(dk)
    np.testing.assert_allclose(loss, ref["loss"], rtol=L_REL, atol=L_ABS)
    # a dense row sums every prior key (up to 4096 here, where the sparse stage sums at most
    # 2048): per row rel-L2 <= 2e-3 and, element by element, a floor of 1e-3 of the tensor's
    # largest element (the sums cancel further over more keys)
    for i in range(n):
        assert _rel_l2(dw[i], ref["dw"][i]) <= G_REL_L2, ("dw", rows[i])
        assert _rel_l2(dq[i], ref["dq"][i]) <= G_REL_L2, ("dq", rows[i])
    assert _rel_l2(dk[ref["dk_rows"]], ref["dk"]) <= G_REL_L2
    _check_elementwise(dw, ref["dw"], "dw", floor=DENSE_FLOOR)
    _check_elementwise(dq, ref["dq"], "dq", floor=DENSE_FLOOR)
    _check_elementwise(dk[ref["dk_rows"]], ref["dk"], "dk", floor=DENSE_FLOOR)
    untouched = np.setdiff1d(np.arange(dk.shape[0]), ref["dk_rows"])
    assert not dk[untouched].any()


def test_dense_warmup_full_dims_4096_rows(dsa):
    """The warm-up stage on a 4096-row sequence at full shapes: rows around pos + 1 = topk and
    at the end of the sequence, where every row has more than topk prior keys."""
    wl = make_prefill(23, [4096], FULL, needles=8, device="cuda")
    _dense_case(dsa, wl, 2040, 16)
    _dense_case(dsa, wl, 4088, 8)


def test_dense_warmup_small_shape(dsa):
    """The same at the small shapes (topk 64, rows of up to 1024 keys: the CUDA-core backward)."""
    wl = make_config(1, device="cuda")
    _dense_case(dsa, wl, 980, 44)
    _dense_case(dsa, wl, 30, 40)
