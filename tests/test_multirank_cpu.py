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


# ------------------------------------------------------------------ sharded prefill (2 ranks)

def _shard_worker(rank, world, port, out_dir):
    """One rank of a prefill split by query rows: its own key-side rows go through the
    all-gather (gloo), and its query rows are computed by the oracle on the gathered keys."""
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}")
    try:
        import sys
        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        import oracle
        from dsa_workloads import make_prefill, TINY
        from sparse_attention_long_04_b200 import shard
        wl = make_prefill(71, [300, 517, 90], TINY, needles=8, device="cpu")
        ranges = shard.split_rows(wl.seqlens, wl.dims, world)
        rb, n = ranges[rank]
        sl = slice(rb, rb + n)
        # this rank starts with its own rows only; the others are destroyed before the exchange
        own = (wl.k_idx[sl].clone(), wl.k_scale[sl].clone(), wl.kv[sl].clone())
        full = (wl.k_idx.clone(), wl.k_scale.clone(), wl.kv.clone())
        wl.k_idx.fill_(0xFF)
        wl.k_scale.fill_(float("nan"))
        wl.kv.fill_(float("nan"))
        k_idx, k_scale, kv = shard.gather_keys(*own, ranges)
        same = [bool(torch.equal(a.view(torch.uint8), b.view(torch.uint8)))
                for a, b in zip((k_idx, k_scale, kv), full)]
        wl.k_idx, wl.k_scale, wl.kv = k_idx, k_scale, kv
        rows = list(range(rb, rb + n))[:: max(1, n // 40)]
        _, idx, o, lse = oracle.forward_rows(wl, rows)
        np.save(os.path.join(out_dir, f"srows{rank}.npy"), np.array(rows))
        np.save(os.path.join(out_dir, f"sidx{rank}.npy"), idx)
        np.save(os.path.join(out_dir, f"so{rank}.npy"), o)
        np.save(os.path.join(out_dir, f"slse{rank}.npy"), lse)
        import json
        with open(os.path.join(out_dir, f"sres{rank}.json"), "w") as f:
            json.dump({"ranges": ranges, "same": same}, f)
    finally:
        dist.destroy_process_group()


def test_sharded_prefill_two_ranks_gloo(tmp_path):
    port = _free_port()
    mp.start_processes(_shard_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    import json
    import oracle
    from dsa_workloads import make_prefill, TINY
    res = [json.load(open(tmp_path / f"sres{r}.json")) for r in (0, 1)]
    assert res[0]["ranges"] == res[1]["ranges"]
    (b0, n0), (b1, n1) = res[0]["ranges"]
    assert b0 == 0 and b1 == n0 and n0 + n1 == 907 and n0 > 0 and n1 > 0
    assert res[0]["same"] == [True, True, True] and res[1]["same"] == [True, True, True]
    wl = make_prefill(71, [300, 517, 90], TINY, needles=8, device="cpu")
    for rank in (0, 1):
        rows = np.load(tmp_path / f"srows{rank}.npy").tolist()
        _, idx, o, lse = oracle.forward_rows(wl, rows)          # single process, all keys
        assert np.array_equal(np.load(tmp_path / f"sidx{rank}.npy"), idx)
        assert np.array_equal(np.load(tmp_path / f"so{rank}.npy"), o)
        assert np.array_equal(np.load(tmp_path / f"slse{rank}.npy"), lse)


def test_split_rows_covers_and_balances():
    """The prefill row split: contiguous ranges covering every packed row once, whose modelled
    work differs from the ideal share by at most one row's work."""
    from sparse_attention_long_04_b200 import shard
    from dsa_workloads import CONFIGS, FULL
    seqlens = CONFIGS[5]["seqlens"]
    a = FULL["h_idx"] * FULL["d_idx"]
    b = 2 * FULL["h"] * (FULL["d_qk"] + FULL["d_v"])
    K = FULL["topk"]
    cost = []
    for L in seqlens:
        p = np.arange(L, dtype=np.float64)
        cost.append(a * (p + 1) + b * np.minimum(p + 1, K))
    cost = np.concatenate(cost)
    for world in (1, 2, 3, 4, 8):
        ranges = shard.split_rows(seqlens, FULL, world)
        assert ranges[0][0] == 0 and sum(n for _, n in ranges) == len(cost)
        for (r0, n0), (r1, _) in zip(ranges, ranges[1:]):
            assert r0 + n0 == r1
        share = cost.sum() / world
        for r0, n in ranges:
            assert abs(cost[r0:r0 + n].sum() - share) <= 2 * cost.max()


# ------------------------------------------------- the bench's timed loop on two ranks (stubbed)

class _WallEvent:
    def __init__(self):
        self.t = None

    def record(self, stream=None):
        import time
        self.t = time.perf_counter()

    def elapsed_time(self, other):
        return (other.t - self.t) * 1e3


class _WallTimer:
    event = staticmethod(_WallEvent)

    @staticmethod
    def sync():
        pass


class _FakeDsa:
    DSA_OK = 0

    @staticmethod
    def dsa_read_device_status(status, stream=None):
        return 0, 0

    @staticmethod
    def check(st, what=""):
        assert st == 0, what


class _FakeStep:
    """Stands in for the three kernel launches: rank 1 is slower than rank 0."""

    def __init__(self, rank):
        self.dsa, self.status, self.stream, self.rank = _FakeDsa(), None, None, rank
        self.calls = 0

    def __call__(self, ev=None):
        import time
        self.calls += 1
        for j in range(3):
            if ev is not None:
                ev[j].record()
            time.sleep(0.001 * (1 + self.rank))
        if ev is not None:
            ev[3].record()


def _bench_worker(rank, world, port, out_dir):
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}")
    try:
        import sys
        import types
        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        import bench
        step = _FakeStep(rank)
        args = types.SimpleNamespace(warmup=3, steps=4)
        ms, per_kernel, _ = bench.time_decode(args, _FakeDsa(), step, world, torch.device("cpu"),
                                              timer=_WallTimer)
        import json
        with open(os.path.join(out_dir, f"b{rank}.json"), "w") as f:
            json.dump({"ms": ms, "per_kernel": per_kernel, "calls": step.calls}, f)
    finally:
        dist.destroy_process_group()


def test_bench_timed_loop_two_ranks_gloo(tmp_path):
    """bench.time_decode on two gloo ranks with the kernels stubbed: W warm-up + K timed steps on
    every rank, barriers around the timed region, the job time is the slower rank's on both, and
    the per-stage split comes from K more steps with events between the stages."""
    port = _free_port()
    mp.start_processes(_bench_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    import json
    r = [json.load(open(tmp_path / f"b{k}.json")) for k in (0, 1)]
    assert r[0]["calls"] == r[1]["calls"] == 3 + 4 + 4
    assert r[0]["ms"] == r[1]["ms"]                     # max over ranks, on both
    assert r[0]["ms"] >= 3 * 2.0 * 0.99                 # rank 1: three 2 ms stages per step
    assert all(x >= 1.9 for x in r[1]["per_kernel"]) and all(x >= 0.9 for x in r[0]["per_kernel"])
