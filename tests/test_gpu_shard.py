"""The building block of the prefill split across GPUs (dsa_forward_rows) on one GPU: every
rank's range of query rows, computed from local copies of that range's query-side arrays and the
full key-side arrays (what the all-gather gives each rank), equals dsa_forward on the same rows
bit for bit: the selection, the output and the LSE.  The ranks are emulated one after another on
the one GPU (no rank waits on another).  Decode row ranges (sequence ranges) are checked the same
way."""
import numpy as np
import pytest
import torch

from dsa_workloads import FULL, TINY, make_decode, make_prefill
from tests.parity import to_np

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_04_b200 as m
    return m


def _full(dsa, wl):
    f = dsa.Forward(wl, keep_idx=True)
    assert f() == dsa.DSA_OK
    torch.cuda.synchronize()
    assert int(f.status.item()) == 0
    return to_np(f.idx), f.out.clone(), f.lse.clone()


def _ranks(dsa, wl, ranges, keep_idx):
    from sparse_attention_long_04_b200 import shard
    pb = dsa.problem_of(wl)
    res = []
    for rb, n in ranges:
        sl = slice(rb, rb + n)
        part = shard.ShardForward(dsa, pb, rb, n, wl.q_idx[sl].clone(), wl.q_scale[sl].clone(),
                                  wl.w[sl].clone(), wl.q[sl].clone(), keep_idx=keep_idx)
        assert part(wl.k_idx, wl.k_scale, wl.kv) == dsa.DSA_OK
        torch.cuda.synchronize()
        assert int(part.status.item()) == 0
        res.append((rb, n, part))
    return res


@pytest.mark.parametrize("dims,lens", [(FULL, [3000, 700, 2100]), (TINY, [1024, 77, 300])])
def test_prefill_row_ranges_equal_the_whole_forward(dsa, dims, lens):
    from sparse_attention_long_04_b200 import shard
    wl = make_prefill(81, lens, dims, needles=8, device="cuda")
    idx, out, lse = _full(dsa, wl)
    for world in (2, 3):
        ranges = shard.split_rows(wl.seqlens, wl.dims, world)
        for rb, n, part in _ranks(dsa, wl, ranges, keep_idx=True):
            assert np.array_equal(to_np(part.idx), idx[rb:rb + n]), (world, rb)
            assert torch.equal(part.out, out[rb:rb + n]), (world, rb)
            assert torch.equal(part.lse, lse[rb:rb + n]), (world, rb)
    # without kept indices the first rows run dense attention: the same outputs
    f = dsa.Forward(wl, keep_idx=False)
    assert f() == dsa.DSA_OK
    ranges = shard.split_rows(wl.seqlens, wl.dims, 3)
    for rb, n, part in _ranks(dsa, wl, ranges, keep_idx=False):
        assert torch.equal(part.out, f.out[rb:rb + n]), rb
        assert torch.equal(part.lse, f.lse[rb:rb + n]), rb


def test_decode_row_ranges_equal_the_whole_forward(dsa):
    wl = make_decode(82, 6, [9000, 2049, 300, 131072, 4096, 1], FULL, boost=0.01, paged=True,
                     device="cuda", scale_layout="interleaved")
    idx, out, lse = _full(dsa, wl)
    for ranges in ([(0, 2), (2, 4)], [(0, 1), (1, 1), (2, 3), (5, 1)]):
        for rb, n, part in _ranks(dsa, wl, ranges, keep_idx=True):
            assert np.array_equal(to_np(part.idx), idx[rb:rb + n]), rb
            # a range of fewer sequences may split the attention differently: same selection,
            # outputs within the attention tolerance of the whole batch's
            o1, o2 = part.out.float(), out[rb:rb + n].float()
            assert (o1 - o2).abs().max().item() <= 2e-2
            assert (part.lse - lse[rb:rb + n]).abs().max().item() <= 1e-3
