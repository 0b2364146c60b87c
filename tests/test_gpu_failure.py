"""Failure detection on the GPU without a fault: a wait that nothing completes ends after its
limit, reports a timeout through the device status word, and leaves the context usable."""
import time

import numpy as np
import pytest
import torch

import oracle
from dsa_workloads import TINY, make_decode
from tests.parity import to_np

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_04_b200 as m
    return m


def test_bounded_wait_times_out_and_context_survives(dsa):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert dsa.dsa_selftest_wait_timeout(status, 0) == dsa.DSA_OK
    st, raw = dsa.dsa_read_device_status(status, 0)
    waited = time.perf_counter() - t0
    assert st == dsa.DSA_ERR_TIMEOUT and raw == dsa.DSA_DEVICE_TIMEOUT
    assert 1.0 < waited < 30.0                        # the 2 s limit, not an early exit
    # the context still runs work: a cache append, checked bit for bit against the oracle
    wl = make_decode(41, 3, [5, 64, 300], dict(TINY), boost=0.0, paged=False, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(4)
    k_new = torch.randn(3, wl.dims["d_idx"], generator=g, device="cuda")
    kv_new = torch.randn(3, wl.dims["d_qk"], generator=g, device="cuda").to(torch.bfloat16)
    ref = oracle.cache_append(wl.k_idx, wl.k_scale, wl.kv, wl.seq_lens, wl.block_table,
                              wl.max_seqlen, k_new, kv_new)
    status.zero_()
    assert dsa.dsa_cache_append(dsa.problem_of(wl), k_new, kv_new, wl.k_idx, wl.k_scale, wl.kv,
                                status, 0) == dsa.DSA_OK
    assert dsa.dsa_read_device_status(status, 0) == (dsa.DSA_OK, 0)
    assert np.array_equal(to_np(wl.k_idx.view(torch.uint8)), ref[0])
    assert np.array_equal(to_np(wl.k_scale), ref[1])
    assert np.array_equal(to_np(wl.kv.view(torch.int16)).view(np.uint16), ref[2])
