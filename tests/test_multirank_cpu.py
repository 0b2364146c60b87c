"""The N > 1 path on CPU: two ranks under the gloo backend (no GPU).

Decode shards by sequence and prefill by whole problems, with no collective on the data path:
every rank draws its own batch (its own seed), the job's time is the slowest rank's, and the
whole-job value counts every rank's units.  These tests run the host-side logic that
`bench.py --gpus N` uses on two real ranks, and check that splitting the rows of one problem
between ranks gives exactly the single-process results (the oracle stands in for the kernels).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}")
    try:
        import sys
        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        import bench
        import oracle
        from dsa_workloads import make_config

        res = {}
        # 1. every rank's batch is its own (weak scaling) and reproducible
        seed = bench.rank_seed(1, rank)
        wl = make_config(1, device="cpu", seed=seed)
        res["seed"] = seed
        res["q_sum"] = float(wl.q_idx.view(torch.uint8).double().sum())
        # 2. the job time is the slowest rank's, on every rank
        ms = [3.0, 7.5][rank]
        res["max_ms"] = bench.max_over_ranks(ms, world, torch.device("cpu"))
        res["value"] = bench.weak_value(world, 64, res["max_ms"])
        # 3. a problem's rows split across ranks: each rank computes its own rows with no
        #    exchange; the gathered result equals the single-process one
        wl0 = make_config(1, device="cpu", seed=bench.rank_seed(1, 0))
        rows = list(range(rank, 96, world))            # rows 0..95, interleaved
        _, idx, o, lse = oracle.forward_rows(wl0, rows)
        np.save(os.path.join(out_dir, f"rows{rank}.npy"), np.array(rows))
        np.save(os.path.join(out_dir, f"idx{rank}.npy"), idx)
        np.save(os.path.join(out_dir, f"lse{rank}.npy"), lse)
        np.save(os.path.join(out_dir, f"o{rank}.npy"), o)
        dist.barrier()
        import json
        with open(os.path.join(out_dir, f"res{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    import json
    r0 = json.load(open(tmp_path / "res0.json"))
    r1 = json.load(open(tmp_path / "res1.json"))
    assert r0["seed"] != r1["seed"]
    assert r0["q_sum"] != r1["q_sum"]                 # different batches per rank
    assert r0["max_ms"] == r1["max_ms"] == 7.5        # max over ranks, on both
    assert r0["value"] == pytest.approx(2 * 64 / 7.5e-3)

    import oracle
    import bench
    from dsa_workloads import make_config
    wl0 = make_config(1, device="cpu", seed=bench.rank_seed(1, 0))
    all_rows = list(range(96))
    _, idx, o, lse = oracle.forward_rows(wl0, all_rows)
    for rank in (0, 1):
        rows = np.load(tmp_path / f"rows{rank}.npy")
        assert np.array_equal(np.load(tmp_path / f"idx{rank}.npy"), idx[rows])
        assert np.array_equal(np.load(tmp_path / f"lse{rank}.npy"), lse[rows])
        assert np.array_equal(np.load(tmp_path / f"o{rank}.npy"), o[rows])


def test_bench_work_models():
    """The bench's FLOP counts and the KL backward roofline, on hand-countable cases."""
    import bench
    d = dict(h_idx=2, d_idx=4, topk=3, h=5, d_qk=6, d_v=4)
    # one sequence of 5 rows, k = 3: selected (row, key) pairs = 1 + 2 + 3 + 3 + 3 = 12
    f_t, f_b = bench.train_flops([5], d)
    assert f_t == 2 * 5 * 6 * 12 and f_b == 3 * 2 * 2 * 4 * 12
    roof = bench.kl_backward_roofline(3e12, 2.0, 1000.0)
    # 1e12 e4m3 FLOP at 2000 TF/s + 2e12 bf16 FLOP at 1000 TF/s = 0.5 ms + 2 ms
    assert roof["ideal_ms"] == pytest.approx(2.5) and roof["frac"] == pytest.approx(1.25)
    assert roof["achieved"] == pytest.approx(1500.0) and roof["bound"] == "tensor"
