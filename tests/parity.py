"""Acceptance checks shared by the GPU parity tests (CUDA path vs the CPU oracle).

Tolerances:
  indexer    |S_gpu - S_ref| <= 1e-3 |S_ref| + 1e-5 max_s S_ref[t, :]   (fp32 accumulation of
             exact fp8 products against the oracle's fp64; the absolute floor covers scores that
             cancel to ~0)
  top-k      (i) the oracle's selector applied to the GPU's own fp32 scores picks exactly the
             GPU's set; (ii) against the oracle's scores, >= 99.9 % of the selected indices
             agree and every disagreement scores within the indexer tolerance of the oracle's
             k-th score (the tolerance at that k-th score, once: not the sum of the two scores'
             tolerances that would bound a swap in the worst case)
  attention  per row rel-L2 <= 5e-3 and max-abs <= 2e-2 of O against the fp64 oracle on the
             GPU's index set; |LSE_gpu - LSE_ref| <= 1e-3
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

IDX_REL, IDX_FLOOR = 1e-3, 1e-5
ATT_REL_L2, ATT_MAX_ABS, LSE_ABS = 5e-3, 2e-2, 1e-3


def check_scores(gpu_row: np.ndarray, ref_row: np.ndarray, what=""):
    gpu_row = np.asarray(gpu_row, np.float64)
    assert gpu_row.shape == ref_row.shape, what
    tol = IDX_REL * np.abs(ref_row) + IDX_FLOOR * max(float(ref_row.max(initial=0.0)), 1e-30)
    err = np.abs(gpu_row - ref_row)
    bad = np.nonzero(err > tol)[0]
    assert len(bad) == 0, (f"{what}: {len(bad)} scores out of tolerance, first s={bad[:5]} "
                           f"gpu={gpu_row[bad[:5]]} ref={ref_row[bad[:5]]}")


def check_topk_layout(idx_row: np.ndarray, n_valid: int, k: int, what=""):
    valid = idx_row[idx_row >= 0]
    assert len(valid) == min(n_valid, k), f"{what}: {len(valid)} selected, expected {min(n_valid, k)}"
    assert (idx_row[len(valid):] == -1).all(), f"{what}: -1 padding not at the end"
    assert (np.diff(valid) > 0).all(), f"{what}: indices not strictly increasing"
    assert valid.min(initial=0) >= 0 and valid.max(initial=0) < n_valid, what


def check_topk_exact(idx_row: np.ndarray, gpu_scores_row: np.ndarray, k: int, what=""):
    """The oracle's selector on the GPU's own scores picks the GPU's set, bit for bit."""
    n = len(gpu_scores_row)
    check_topk_layout(idx_row, n, k, what)
    ref = oracle.topk_rows([np.asarray(gpu_scores_row, np.float64)], k)[0]
    assert np.array_equal(np.sort(ref[ref >= 0]), idx_row[idx_row >= 0]), what


def topk_overlap(idx_rows, ref_scores_rows, k):
    """(overlap fraction, list of mismatch violations) against the oracle's own scores."""
    ref_idx = oracle.topk_rows(ref_scores_rows, k)
    hit = tot = 0
    viol = []
    for g, r, s in zip(idx_rows, ref_idx, ref_scores_rows):
        gs, rs = set(g[g >= 0].tolist()), set(r[r >= 0].tolist())
        hit += len(gs & rs)
        tot += len(rs)
        if gs != rs:
            tau = min(s[list(rs)])
            tol = IDX_REL * abs(tau) + IDX_FLOOR * s.max()
            for x in gs ^ rs:
                if abs(s[x] - tau) > tol:
                    viol.append((x, s[x], tau))
    return (hit / tot if tot else 1.0), viol


def check_attention(out_gpu, lse_gpu, out_ref, lse_ref, n_heads: int, what=""):
    o = np.asarray(out_gpu, np.float64)[:n_heads]
    r = np.asarray(out_ref, np.float64)[:n_heads]
    num = np.linalg.norm(o - r)
    den = max(np.linalg.norm(r), 1e-30)
    assert num / den <= ATT_REL_L2, f"{what}: rel-L2 {num / den:.3e}"
    assert np.abs(o - r).max(initial=0.0) <= ATT_MAX_ABS, f"{what}: max-abs {np.abs(o - r).max():.3e}"
    lg = np.asarray(lse_gpu, np.float64)[:n_heads]
    lr = np.asarray(lse_ref, np.float64)[:n_heads]
    fin = np.isfinite(lr)
    assert np.array_equal(fin, np.isfinite(lg)), f"{what}: -inf pattern differs"
    if fin.any():
        assert np.abs(lg[fin] - lr[fin]).max() <= LSE_ABS, (
            f"{what}: LSE err {np.abs(lg[fin] - lr[fin]).max():.3e}")


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy()


def n_valid_of(wl, row: int) -> int:
    geo = oracle.Geometry.of(wl)
    return geo.row_seq_pos(row)[1] + 1
