"""The allocation-free sparse MLA entry point against the regular one.

dsa_sparse_mla_fwd_noalloc exists for callers that may not allocate device memory at all (work
recorded into a CUDA graph, runtimes that own every byte through a fixed pool, plugins whose host
forbids allocator calls on the hot path).  It keeps its split-KV partials in a scratch array built
into the library instead of a caller workspace, choosing a split count whose partials fit it.  This
test runs it on decode batches of 3 rows (split, the partials in the built-in scratch), 37 rows
(the largest split batch that still fits), 40 rows (whose unconstrained split would not fit, so it
runs with fewer splits) and 64 rows (unsplit), twice in a row with different selections, and
compares each result with dsa_sparse_mla_fwd given a normal workspace, within the attention
tolerance of the parity tests.  The file is named so that pytest collects it last.
"""
import pytest
import torch

from dsa_workloads import FULL, make_decode
from tests.parity import check_attention, to_np

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _selection(lens, k, seed):
    g = torch.Generator().manual_seed(seed)
    idx = torch.full((len(lens), k), -1, dtype=torch.int32)
    for i, n in enumerate(lens):
        m = min(n, k)
        idx[i, :m] = torch.randperm(n, generator=g)[:m].to(torch.int32)
    return idx.cuda()


def _lens(rows):
    base = [6000, 2048, 300]
    return base if rows == 3 else [base[i % 3] + 37 * i for i in range(rows)]


@pytest.mark.parametrize("rows", [3, 37, 40, 64])
def test_noalloc_matches_workspace_entry_point_on_two_calls(rows):
    import sparse_attention_long_04_b200 as dsa
    lens = _lens(rows)
    wl = make_decode(41, len(lens), lens, FULL, boost=0.0, paged=True, device="cuda")
    pb = dsa.problem_of(wl)
    ws_bytes = dsa.dsa_sparse_mla_workspace_size(pb, rows)
    if rows == 3:
        assert 0 < ws_bytes <= dsa.NOALLOC_SCRATCH_BYTES      # the path that needs scratch
    d = wl.dims
    for call, seed in enumerate((1, 2)):
        idx = _selection(lens, d["topk"], seed)
        ref_out = torch.full((rows, d["h"], d["d_v"]), float("nan"), dtype=torch.bfloat16,
                             device="cuda")
        ref_lse = torch.full((rows, d["h"]), float("nan"), device="cuda")
        ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
        assert dsa.dsa_sparse_mla_fwd(pb, wl.q, wl.kv, idx, 0, rows, ref_out, ref_lse, ws,
                                      ws_bytes) == dsa.DSA_OK
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        st = dsa.dsa_sparse_mla_fwd_noalloc(pb, wl.q, wl.kv, idx, 0, rows, out, lse, status)
        assert st == dsa.DSA_OK, dsa.status_string(st)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        o, l, ro, rl = to_np(out), to_np(lse), to_np(ref_out), to_np(ref_lse)
        for r in range(rows):
            check_attention(o[r], l[r], ro[r], rl[r], d["h"], f"call {call} row {r}")
