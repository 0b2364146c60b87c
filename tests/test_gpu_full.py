"""Full-size parity: the four full-shape workloads at their real sizes, run through dsa_forward
(the launch configuration the benchmark times), checked against the oracle on seeded samples
of rows.

  decode_B32_N32k         all 32 rows
  decode_B64_N128k_paged  all 64 rows
  prefill_L16k            512 sampled rows + every row with position < 64
  prefill_varlen_T276480  256 sampled rows per sequence (+ positions < 64 of the first one)

Per sampled row: the selected set against the oracle's own scores (>= 99.9 % overlap, every
miss within the score tolerance of the k-th score) and the attention output / LSE against the
fp64 oracle on the GPU's selection.  On a subset of rows the indexer scores themselves are
checked, and the top-k is checked bit-exactly on the GPU's own scores.
"""
import numpy as np
import pytest
import torch

import oracle
from dsa_workloads import make_config, sample_rows
from tests.parity import (check_attention, check_scores, check_topk_exact, check_topk_layout,
                          n_valid_of, to_np, topk_overlap)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

SAMPLES = {2: dict(all_rows=True), 3: dict(all_rows=True),
           4: dict(per_seq=512, first=64), 5: dict(per_seq=256, first=64)}


def _rows(wl, cfg):
    s = SAMPLES[cfg]
    if s.get("all_rows"):
        return list(range(wl.total_rows))
    rows = sample_rows(wl, s["per_seq"])
    return sorted(set(rows) | set(range(min(s["first"], wl.seqlens[0]))))


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_forward_full_size_sampled_rows(cfg):
    import sparse_attention_long_04_b200 as dsa
    wl = make_config(cfg, device="cuda")
    f = dsa.Forward(wl)
    st = f()
    assert st == dsa.DSA_OK, dsa.status_string(st)
    torch.cuda.synchronize()
    st, raw = dsa.dsa_read_device_status(f.status)
    assert st == dsa.DSA_OK, raw
    rows = _rows(wl, cfg)
    k = wl.dims["topk"]
    ref_scores = oracle.indexer_rows(wl, rows)
    gidx = to_np(f.idx.index_select(0, torch.tensor(rows, device="cuda")))
    for i, r in enumerate(rows):
        check_topk_layout(gidx[i], n_valid_of(wl, r), k, f"row {r}")
    frac, viol = topk_overlap(list(gidx), [ref_scores[r] for r in rows], k)
    assert frac >= 0.999 and not viol, (frac, viol[:5])
    ro, rl = oracle.sparse_mla_rows(wl, rows, gidx)
    sel = torch.tensor(rows, device="cuda")
    o = to_np(f.out.index_select(0, sel))
    l = to_np(f.lse.index_select(0, sel))
    for i, r in enumerate(rows):
        check_attention(o[i], l[i], ro[i], rl[i], wl.dims["h"], f"row {r}")

    # indexer scores and bit-exact selection on the GPU's own scores, on a subset of rows
    pb = dsa.problem_of(wl)
    sub = rows[:: max(1, len(rows) // 16)]
    for r in sub:
        n = n_valid_of(wl, r)
        ld = (n + 3) // 4 * 4
        sc = torch.full((1, ld), float("nan"), device="cuda")
        assert dsa.dsa_indexer_scores(pb, wl.q_idx, wl.q_scale, wl.w, wl.k_idx, wl.k_scale, r,
                                      1, sc, ld) == dsa.DSA_OK
        ix = torch.empty(1, k, dtype=torch.int32, device="cuda")
        assert dsa.dsa_topk(pb, sc, ld, r, 1, ix) == dsa.DSA_OK
        torch.cuda.synchronize()
        s_np = to_np(sc)[0, :n]
        check_scores(s_np, ref_scores[r], f"row {r}")
        check_topk_exact(to_np(ix)[0], s_np, k, f"row {r}")
