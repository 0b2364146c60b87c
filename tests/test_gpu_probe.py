"""The diagnostics.  The distributed-shared-memory probe (dsa_probe_dsmem): every word lands as
written, with one cluster alone and with clusters on every SM, and the timing it returns is
positive.  The key-page stream probe (dsa_probe_page_stream): it reads every block of a
shuffled list and counts exactly the ids outside the buffer, which it skips."""
import pytest
import torch

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("clusters", [1, 74])
def test_dsmem_probe_exchanges_every_word(clusters):
    import sparse_attention_long_04_b200 as dsa
    ns = torch.zeros(clusters, dtype=torch.int64, device="cuda")
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert dsa.dsa_probe_dsmem(clusters, 32 * 1024, 16, ns, bad) == dsa.DSA_OK
    torch.cuda.synchronize()
    assert int(bad.item()) == 0
    assert bool((ns > 0).all())


@pytest.mark.parametrize("ctas_per_sm", [1, 2, 8])
def test_page_stream_probe_counts_bad_ids(ctas_per_sm):
    import sparse_attention_long_04_b200 as dsa
    nblk, bb = 64, 64 * (128 + 4)               # pages of 64 rows of 128 B, then 64 scales
    blocks = torch.zeros(nblk, bb, dtype=torch.uint8, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(5)
    ids = torch.randperm(nblk, generator=g, device="cuda").to(torch.int32).repeat(10)
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert dsa.dsa_probe_page_stream(blocks, ids, nblk, 128, ctas_per_sm, bad) == dsa.DSA_OK
    torch.cuda.synchronize()
    assert int(bad.item()) == 0
    ids[5], ids[77], ids[600] = -1, nblk, 1 << 30
    assert dsa.dsa_probe_page_stream(blocks, ids, nblk, 128, ctas_per_sm, bad) == dsa.DSA_OK
    torch.cuda.synchronize()
    assert int(bad.item()) == 3
