"""The distributed-shared-memory probe (dsa_probe_dsmem): every word lands as written, with one
cluster alone and with clusters on every SM, and the timing it returns is positive."""
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
