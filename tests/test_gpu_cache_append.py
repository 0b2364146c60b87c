"""Decode cache append on the GPU against the oracle, bit for bit: the e4m3 codes and scales of
the new tokens' indexer keys, their latent rows, and every other cache row left untouched."""
import numpy as np
import pytest
import torch

import oracle
from dsa_workloads import FULL, TINY, make_config, make_decode
from tests.parity import to_np

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_04_b200 as m
    return m


def _new_tokens(wl, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    B, d = wl.batch, wl.dims
    k_new = torch.randn(B, d["d_idx"], generator=g, device="cuda") * 3.0
    k_new[0, :5] = 0.0                                  # zeros in a row
    kv_new = torch.randn(B, d["d_qk"], generator=g, device="cuda").to(torch.bfloat16)
    return k_new, kv_new


def _append(dsa, wl, k_new, kv_new):
    pb = dsa.problem_of(wl)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = dsa.dsa_cache_append(pb, k_new, kv_new, wl.k_idx, wl.k_scale, wl.kv, status)
    assert st == dsa.DSA_OK, dsa.status_string(st)
    torch.cuda.synchronize()
    return int(status.item())


@pytest.mark.parametrize("paged,dims,layout", [(True, FULL, "separate"),
                                               (True, FULL, "interleaved"),
                                               (False, dict(TINY), "separate")])
def test_cache_append_whole_caches(dsa, paged, dims, layout):
    lens = [700, 64, 1, 130, 4096]
    wl = make_decode(31, len(lens), lens, dims, boost=0.0, paged=paged, device="cuda",
                     total_blocks=400 if paged else None, scale_layout=layout)
    k_new, kv_new = _new_tokens(wl, 7)
    ref = oracle.cache_append(wl.k_idx, wl.k_scale, wl.kv, wl.seq_lens, wl.block_table,
                              wl.max_seqlen, k_new, kv_new)
    assert _append(dsa, wl, k_new, kv_new) == 0
    assert not ref[3].any()
    assert np.array_equal(to_np(wl.k_idx.view(torch.uint8)), ref[0])
    if wl.k_scale is not None:
        assert np.array_equal(to_np(wl.k_scale), ref[1])
    assert np.array_equal(to_np(wl.kv.view(torch.int16)).view(np.uint16), ref[2])


def test_cache_append_bad_entries_skipped(dsa):
    lens = [300, 64, 130]
    wl = make_decode(32, 3, lens, FULL, boost=0.0, paged=True, device="cuda", total_blocks=20)
    wl.block_table[1, 0] = -1                           # the new token's block is invalid
    wl.seq_lens[2] = wl.max_seqlen + 1                  # a length past the caches
    k_new, kv_new = _new_tokens(wl, 8)
    ref = oracle.cache_append(wl.k_idx, wl.k_scale, wl.kv, wl.seq_lens, wl.block_table,
                              wl.max_seqlen, k_new, kv_new)
    assert list(ref[3]) == [False, True, True]
    status = _append(dsa, wl, k_new, kv_new)
    assert status & dsa.DSA_DEVICE_BAD_INDEX
    assert np.array_equal(to_np(wl.k_idx.view(torch.uint8)), ref[0])
    assert np.array_equal(to_np(wl.k_scale), ref[1])
    assert np.array_equal(to_np(wl.kv.view(torch.int16)).view(np.uint16), ref[2])


def test_cache_append_full_size_decode_128k(dsa):
    """decode_B64_N128k_paged: the 64 appended rows bit for bit, and 2000 sampled untouched
    rows unchanged."""
    wl = make_config(3, device="cuda")
    k_new, kv_new = _new_tokens(wl, 9)
    geo = oracle.Geometry.of(wl)
    rows = np.array([int(geo.phys(b, np.array([n - 1]))[0]) for b, n in enumerate(wl.seqlens)])
    g = np.random.default_rng(3)
    others = np.setdiff1d(g.integers(0, wl.kv.shape[0], 2000), rows)
    sel = torch.tensor(others, device="cuda")
    before_k = oracle.key_rows(wl, others)             # this workload's key blocks hold scales
    before_kv = wl.kv.index_select(0, sel).clone()
    assert _append(dsa, wl, k_new, kv_new) == 0
    codes, scales = oracle.quantize_e4m3(k_new)
    got_c, got_s = oracle.key_rows(wl, rows)
    assert np.array_equal(got_c, codes) and np.array_equal(got_s, scales)
    r = torch.tensor(rows, device="cuda")
    assert torch.equal(wl.kv.index_select(0, r), kv_new)
    after_k = oracle.key_rows(wl, others)
    assert np.array_equal(after_k[0], before_k[0]) and np.array_equal(after_k[1], before_k[1])
    assert torch.equal(wl.kv.index_select(0, sel), before_kv)
