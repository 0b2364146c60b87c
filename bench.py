"""Benchmark of the DSA hot path on B200: decode at 128k context (primary line) and varlen
prefill up to 128k (secondary), plus the CPU oracle as the reported baseline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-prefill]

One step = one pass of the whole path (indexer -> top-k -> sparse MLA-MQA) over one batch:
  decode  : 64 sequences x 131072 context, 64-token pages, random block table (one new token
            each); inputs (11 GB of caches) are far larger than L2, so no flush is needed
  prefill : 8 packed causal sequences {4096 ... 131072}, T = 276480 rows
With N > 1 (torchrun) every rank runs its own independent decode batch (weak scaling, no
collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import copy
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DECODE_CFG, PREFILL_CFG = 3, 5
TRAIN_CFG = 4   # the indexer's training step runs on prefill_L16k (one causal 16384-row sequence)
METRIC = "DSA decode tokens/s and prefill tokens/s at 128k ctx; % of HBM/tensor roofline"


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ------------------------------------------------------------------------------ ranks

def rank_seed(cfg: int, rank: int) -> int:
    """Seed of rank `rank`'s own synthetic batch (weak scaling: every rank draws a different
    batch of the same shape)."""
    return 1000 + cfg + 7919 * rank


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time (the job's time); no collective when world == 1."""
    if world <= 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_value(world: int, units_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput: the units all ranks processed per second of the slowest rank."""
    return world * units_per_rank / (ms_per_step / 1e3)


# ------------------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples (every 200 ms) while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            sel = str(device_index)
        self.sel = sel

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.flush()
        self.f.seek(0)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.f.name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------ work model

def decode_algorithmic_bytes(wl):
    """Bytes the decode step must move at minimum: indexer keys + scales of every context token,
    the selected latent rows, the per-token query inputs and the outputs."""
    d = wl.dims
    ctx = sum(wl.seqlens)
    k_i = ctx * (d["d_idx"] + 4)
    sel = sum(min(L, d["topk"]) for L in wl.seqlens) * d["d_qk"] * 2
    q_in = wl.batch * (d["h"] * d["d_qk"] * 2 + d["h_idx"] * (d["d_idx"] + 8))
    out = wl.batch * d["h"] * (d["d_v"] * 2 + 4)
    return dict(indexer=k_i, total=k_i + sel + q_in + out)


def prefill_flops(seqlens, d):
    """Causal algorithmic FLOPs: indexer 2*H_I*D_I per (query, prior key) pair (fp8); attention
    2*H*(D_qk + D_v) per (query, selected key) pair (bf16)."""
    K = d["topk"]
    pairs = sum(L * (L + 1) // 2 for L in seqlens)
    sel = 0
    for L in seqlens:
        m = min(L, K)
        sel += m * (m + 1) // 2 + (L - m) * K
    return (2 * d["h_idx"] * d["d_idx"] * pairs, 2 * d["h"] * (d["d_qk"] + d["d_v"]) * sel)


def train_flops(seqlens, d):
    """Algorithmic FLOPs of one indexer training step on the top-k selection: the target's
    logits, 2*H*D_qk per (query, selected key) (bf16); the backward's three contractions (D,
    dq, dk), 3 * 2*H_I*D_I per (query, selected key) (fp32)."""
    K = d["topk"]
    sel = 0
    for L in seqlens:
        m = min(L, K)
        sel += m * (m + 1) // 2 + (L - m) * K
    return 2 * d["h"] * d["d_qk"] * sel, 3 * 2 * d["h_idx"] * d["d_idx"] * sel


def kl_backward_roofline(flops_3, ms, bf16_tflops):
    """Tensor roofline of the KL backward: of its three contractions (equal FLOPs), D runs in
    e4m3 (peak taken as 2x bf16, the nominal ratio) and dk, dq in bf16.  Returns the roofline
    dict for a launch of `ms` milliseconds."""
    f8, f16 = flops_3 / 3.0, 2.0 * flops_3 / 3.0
    ideal_ms = (f8 / (2.0 * bf16_tflops * 1e12) + f16 / (bf16_tflops * 1e12)) * 1e3
    achieved = flops_3 / (ms / 1e3) / 1e12
    eff_peak = flops_3 / (ideal_ms / 1e3) / 1e12
    return {"kernel": "dsa_indexer_kl_bwd_tc_kernel", "bound": "tensor",
            "achieved": round(achieved, 1), "peak": round(eff_peak, 1), "unit": "TFLOP/s",
            "frac": round(ideal_ms / ms, 4), "flops": int(flops_3),
            "ideal_ms": round(ideal_ms, 3),
            "peak_note": "D in e4m3 at 2x the measured bf16 sustained peak (nominal ratio), dk and "
                         "dq in bf16 at the measured sustained peak; the hi/lo coefficient pairs "
                         "double the bf16 MMA work but count once"}


# ------------------------------------------------------------------------------ our arm

class DecodeStep:
    """The staged decode step on one workload: the indexer counting each row's first radix digit
    as it writes the scores, the top-k starting from those counts, the sparse MLA forward (the
    same kernels dsa_forward runs), with optional CUDA events between the calls."""

    def __init__(self, dsa, wl, stream):
        d = wl.dims
        dev = wl.kv.device
        self.dsa, self.wl, self.stream = dsa, wl, stream
        self.pb = dsa.problem_of(wl)
        B = wl.batch
        self.ld = (wl.max_seqlen + 3) // 4 * 4
        self.scores = torch.empty(B, self.ld, dtype=torch.float32, device=dev)
        self.hist = torch.zeros(B, dsa.TOPK_HIST_BINS, dtype=torch.int32, device=dev)
        self.idx = torch.empty(B, d["topk"], dtype=torch.int32, device=dev)
        self.out = torch.empty(B, d["h"], d["d_v"], dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(B, d["h"], dtype=torch.float32, device=dev)
        self.mla_ws_bytes = dsa.dsa_sparse_mla_workspace_size(self.pb, B)
        self.mla_ws = torch.empty(max(self.mla_ws_bytes, 16), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.launches = 3 + (1 if self.mla_ws_bytes > 0 else 0)

    def __call__(self, ev=None):
        dsa, wl, st, B = self.dsa, self.wl, self.stream, self.wl.batch
        if ev is not None:
            ev[0].record(st)
        dsa.check(dsa.dsa_indexer_scores(self.pb, wl.q_idx, wl.q_scale, wl.w, wl.k_idx,
                                         wl.k_scale, 0, B, self.scores, self.ld, self.status, st,
                                         hist=self.hist), "indexer")
        if ev is not None:
            ev[1].record(st)
        dsa.check(dsa.dsa_topk(self.pb, self.scores, self.ld, 0, B, self.idx, self.status, st,
                               hist=self.hist), "topk")
        if ev is not None:
            ev[2].record(st)
        dsa.check(dsa.dsa_sparse_mla_fwd(self.pb, wl.q, wl.kv, self.idx, 0, B, self.out,
                                         self.lse, self.mla_ws, self.mla_ws_bytes, self.status,
                                         st), "sparse_mla")
        if ev is not None:
            ev[3].record(st)


class CudaTimer:
    """CUDA events on the launching stream and device synchronisation (the bench's clock)."""

    @staticmethod
    def event():
        return torch.cuda.Event(enable_timing=True)

    @staticmethod
    def sync():
        torch.cuda.synchronize()


def time_decode(args, dsa, step, world, dev, clocks=None, timer=CudaTimer):
    """W warm-up steps, then K timed steps back to back (nothing between them but the launches,
    so each kernel's dependent launch overlaps the previous one's tail), bracketed by a barrier
    and a device synchronisation on both sides; then K more steps with events between the stages
    for the per-kernel split.  Returns (ms per step (max over ranks), mean ms per stage
    [indexer, top-k, sparse MLA], clocks)."""
    stream = step.stream
    for _ in range(args.warmup):
        step()
    timer.sync()
    st, raw = step.dsa.dsa_read_device_status(step.status, stream)
    step.dsa.check(st, "device status after warm-up")
    evs = [[timer.event() for _ in range(4)] for _ in range(args.steps)]
    start, end = timer.event(), timer.event()
    if clocks is not None:
        clocks.start()
        time.sleep(0.25)
    if world > 1:
        torch.distributed.barrier()
    timer.sync()
    start.record(stream)
    for i in range(args.steps):
        step()
    end.record(stream)
    timer.sync()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop() if clocks is not None else None
    ms = start.elapsed_time(end)
    for i in range(args.steps):           # the per-stage split, in a pass of its own
        step(evs[i])
    timer.sync()
    k_ms = [[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3])]
            for e in evs]
    per_kernel = [sum(x[j] for x in k_ms) / len(k_ms) for j in range(3)]
    st, raw = step.dsa.dsa_read_device_status(step.status, stream)
    step.dsa.check(st, "device status after timing")
    return max_over_ranks(ms, world, dev) / args.steps, per_kernel, clk


def decode_rooflines(wl, ms_step, per_kernel, peaks, traffic=None):
    work = decode_algorithmic_bytes(wl)
    idx_gbs = work["indexer"] / (per_kernel[0] / 1e3) / 1e9
    step_gbs = work["total"] / (ms_step / 1e3) / 1e9
    roof = {"kernel": "dsa_indexer_kernel (decode)", "bound": "hbm",
            "achieved": round(idx_gbs, 1), "peak": peaks["hbm"], "unit": "GB/s",
            "frac": round(idx_gbs / peaks["hbm"], 4), "traffic": traffic,
            "peak_source": peaks["source"],
            "algorithmic_bytes_per_launch": work["indexer"]}
    step_roof = {"bound": "hbm", "achieved": round(step_gbs, 1), "unit": "GB/s",
                 "frac": round(step_gbs / peaks["hbm"], 4),
                 "algorithmic_bytes_per_step": work["total"]}
    return roof, step_roof


def run_ours(args, rank, world, local_rank):
    import sparse_attention_long_04_b200 as dsa
    from dsa_workloads import make_config, CONFIGS

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks = read_peaks()
    stream = torch.cuda.current_stream()
    if args.decode_batch:
        from dsa_workloads import make_decode
        c = CONFIGS[DECODE_CFG]
        wl = make_decode(DECODE_CFG, args.decode_batch, c["ctx"],
                         {k: c[k] for k in ("h_idx", "d_idx", "topk", "h", "d_qk", "d_v")},
                         c["boost"], c["paged"], dev, seed=rank_seed(DECODE_CFG, rank),
                         name=f"{c['name']}_B{args.decode_batch}",
                         scale_layout=c.get("scale_layout", "separate"))
    else:
        wl = make_config(DECODE_CFG, device=dev, seed=rank_seed(DECODE_CFG, rank))
    d = wl.dims
    B = wl.batch
    step = DecodeStep(dsa, wl, stream)
    ms_step, per_kernel, clk = time_decode(args, dsa, step, world, dev,
                                           clocks=ClockSampler(local_rank))
    value = weak_value(world, B, ms_step)
    out, lse = step.out, step.lse

    # ---- end to end through the public call, host buffers, copies inside the timed region.
    # Two buffer sets and three streams, as a serving loop runs it: step i+1's inputs go up
    # (host -> device) while step i computes and step i-1's results come down.  Every step
    # still copies all of its inputs from pinned host memory and reads back its out + lse.
    in_keys = ("q", "q_idx", "q_scale", "w", "seq_lens")
    host_in = {k: getattr(wl, k).cpu().pin_memory() for k in in_keys}
    sets = []
    for b in range(2):
        wl_b = copy.copy(wl)
        for k in in_keys:
            setattr(wl_b, k, torch.empty_like(getattr(wl, k)))
        sets.append(dict(wl=wl_b, fwd=dsa.Forward(wl_b, keep_idx=False),
                         out=torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                         lse=torch.empty(lse.shape, dtype=lse.dtype).pin_memory()))
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sets[0]["out"].numel() * 2 + sets[0]["lse"].numel() * 4
    s_up, s_comp, s_down = (torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev),
                            torch.cuda.Stream(device=dev))
    computed = [torch.cuda.Event(), torch.cuda.Event()]
    uploaded = [torch.cuda.Event(), torch.cuda.Event()]
    downloaded = [torch.cuda.Event(), torch.cuda.Event()]

    def e2e_steps(n):
        for i in range(n):
            b = i % 2
            st_b = sets[b]
            if i >= 2:
                s_up.wait_event(computed[b])           # the set's inputs were consumed
            with torch.cuda.stream(s_up):
                for k in in_keys:
                    getattr(st_b["wl"], k).copy_(host_in[k], non_blocking=True)
                uploaded[b].record(s_up)
            s_comp.wait_event(uploaded[b])
            if i >= 2:
                s_comp.wait_event(downloaded[b])       # the set's outputs were read back
            dsa.check(st_b["fwd"](s_comp), "dsa_forward")
            computed[b].record(s_comp)
            s_down.wait_event(computed[b])
            with torch.cuda.stream(s_down):
                st_b["out"].copy_(st_b["fwd"].out, non_blocking=True)
                st_b["lse"].copy_(st_b["fwd"].lse, non_blocking=True)
                downloaded[b].record(s_down)

    e2e_steps(max(2, args.warmup))
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    e2e_steps(args.steps)
    s_down.wait_stream(s_up)
    s_down.wait_stream(s_comp)
    e1.record(s_down)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = weak_value(world, B, e2e_ms / args.steps)
    for st_b in sets:
        st_e, _ = dsa.dsa_read_device_status(st_b["fwd"].status, stream)
        dsa.check(st_e, "e2e device status")
    del sets

    roof, step_roof = decode_rooflines(wl, ms_step, per_kernel, peaks,
                                       traffic=load_traffic("indexer_decode"))
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3+bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "batch": B,
                   "context": wl.max_seqlen, "page": 64, "topk": d["topk"],
                   "indexer": f"{d['h_idx']}x{d['d_idx']} e4m3", "heads": d["h"],
                   "latent": d["d_qk"], "d_v": d["d_v"],
                   "l2": "inputs larger than L2 (11 GB of caches per step)",
                   "parallelism": f"replicas{world}"},
        "roofline": roof,
        "step_roofline": step_roof,
        "kernel_ms": {"indexer": round(per_kernel[0], 4), "topk": round(per_kernel[1], 4),
                      "sparse_mla": round(per_kernel[2], 4)},
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": "per step: new-token inputs (q, q_idx, q_scale, w, seq_lens) copied "
                        "from pinned host memory, dsa_forward, out + lse copied back; the "
                        "paged caches stay resident; two buffer sets on three streams overlap "
                        "step i+1's upload and step i-1's download with step i"},
        "gpu_launches": step.launches * args.steps,
        "clocks": clk,
    }
    line["cache_append"] = time_cache_append(args, dsa, wl, stream, peaks,
                                             cpu_leg=rank == 0 and not args.no_cpu)
    line["probes"] = {"dsmem": probe_dsmem(dsa, dev, stream),
                      "page_stream": probe_page_stream(dsa, wl, dev, stream, roof)}
    if rank == 0 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_seconds)
    del step, out, lse, wl
    torch.cuda.empty_cache()
    if not args.no_extra:
        line["decode_B32_N32k"] = run_decode_extra(args, dsa, dev, stream, peaks, rank, world)
    if not args.no_prefill:
        line["prefill"] = run_prefill(args, dsa, dev, stream, peaks, rank, world, PREFILL_CFG)
        if not args.no_extra:
            line["prefill_L16k"] = run_prefill(args, dsa, dev, stream, peaks, rank, world, 4)
    if not args.no_train:
        line["indexer_train"] = run_indexer_train(args, dsa, dev, stream, peaks, rank, world,
                                                  cpu_leg=rank == 0 and not args.no_cpu)
    return line


def run_decode_extra(args, dsa, dev, stream, peaks, rank, world, cfg=2):
    """decode_B32_N32k: the same staged step on the 32-sequence, 32k-context workload
    (contiguous caches), with its rooflines and the oracle on a sample of its rows."""
    from dsa_workloads import make_config, CONFIGS
    import oracle
    wl = make_config(cfg, device=dev, seed=rank_seed(cfg, rank))
    step = DecodeStep(dsa, wl, stream)
    ms_step, per_kernel, _ = time_decode(args, dsa, step, world, dev)
    roof, step_roof = decode_rooflines(wl, ms_step, per_kernel, peaks)
    res = {"workload": CONFIGS[cfg]["name"], "value": round(weak_value(world, wl.batch, ms_step), 1),
           "unit": "tokens/s", "ms_per_step": round(ms_step, 4), "steps": args.steps,
           "kernel_ms": {"indexer": round(per_kernel[0], 4), "topk": round(per_kernel[1], 4),
                         "sparse_mla": round(per_kernel[2], 4)},
           "roofline": roof, "step_roofline": step_roof,
           "l2": "inputs larger than L2 (2.4 GB of latent rows, 138 MB of indexer keys)",
           "gpu_launches_per_step": step.launches}
    if rank == 0 and not args.no_cpu:
        n = min(wl.batch, oracle.num_threads())
        t0 = time.perf_counter()
        oracle.forward_rows(wl, list(range(n)))
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": round(n / dt, 3), "unit": "tokens/s",
                               "cores": oracle.num_threads(), "kind": "oracle",
                               "sample": f"{n} of {wl.batch} decode rows (full 32768-key "
                                         f"indexer, top-k, fp64 attention per row), {dt:.1f} s"}
    del step, wl
    torch.cuda.empty_cache()
    return res


def prefill_stage_split(dsa, wl, stream, sm_count):
    """One pass over the same row chunks dsa_forward runs (its own chunk plan), through the stage
    calls with CUDA events around each launch: the dense attention of the first topk rows of
    every sequence, then per chunk the indexer (counting the first digit), the top-k (from the
    counts) and the sparse MLA forward.  Returns the summed ms per stage."""
    pb = dsa.problem_of(wl)
    d = wl.dims
    K = d["topk"]
    dev = wl.kv.device
    plan, off = [], 0
    for b, L in enumerate(wl.seqlens):
        rows = dsa.dsa_forward_chunk_rows_for(pb, b, sm_count)
        plan.append((off, L, rows))
        off += L
    ld_max = max((L + 3) // 4 * 4 * rows for _, L, rows in plan if L > K)
    rows_max = max(rows for _, L, rows in plan)
    slab = torch.empty(ld_max, dtype=torch.float32, device=dev)
    hist = torch.zeros(rows_max, dsa.TOPK_HIST_BINS, dtype=torch.int32, device=dev)
    idx = torch.empty(rows_max, K, dtype=torch.int32, device=dev)
    out = torch.empty(wl.total_rows, d["h"], d["d_v"], dtype=torch.bfloat16, device=dev)
    lse = torch.empty(wl.total_rows, d["h"], dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    marks = []   # (stage, start event, end event)

    def timed(stage, fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dsa.check(fn(), stage)
        b.record(stream)
        marks.append((stage, a, b))

    for c0, L, rows in plan:
        nd = min(L, K)
        timed("sparse_mla_dense", lambda: dsa.dsa_sparse_mla_fwd(pb, wl.q, wl.kv, None, c0, nd,
                                                                 out, lse, None, 0, status,
                                                                 stream))
        ld = (L + 3) // 4 * 4
        for r0 in range(nd, L, rows):
            rb, n = c0 + r0, min(rows, L - r0)
            timed("indexer", lambda: dsa.dsa_indexer_scores(pb, wl.q_idx, wl.q_scale, wl.w,
                                                            wl.k_idx, wl.k_scale, rb, n, slab,
                                                            ld, status, stream, hist=hist))
            timed("topk", lambda: dsa.dsa_topk(pb, slab, ld, rb, n, idx, status, stream,
                                               hist=hist))
            timed("sparse_mla", lambda: dsa.dsa_sparse_mla_fwd(pb, wl.q, wl.kv, idx, rb, n, out,
                                                               lse, None, 0, status, stream))
    torch.cuda.synchronize()
    st, _ = dsa.dsa_read_device_status(status, stream)
    dsa.check(st, "staged prefill status")
    split = {}
    for stage, a, b in marks:
        split[stage] = split.get(stage, 0.0) + a.elapsed_time(b)
    return split, len(marks)


def run_prefill_sharded(args, dsa, dev, stream, peaks, rank, world, cfg):
    """N > 1: one prefill problem split over the ranks (strong scaling).  Each rank holds its
    range of query rows and the key-side rows of that range; a step is the all-gather of the
    key-side rows (NCCL) and dsa_forward_rows on the rank's rows.  Time: max over ranks."""
    from dsa_workloads import make_config, CONFIGS
    from sparse_attention_long_04_b200 import shard
    wl = make_config(cfg, device=dev, seed=rank_seed(cfg, 0))      # the same problem everywhere
    pb = dsa.problem_of(wl)
    ranges = shard.split_rows(wl.seqlens, wl.dims, world)
    rb, n = ranges[rank]
    sl = slice(rb, rb + n)
    local_keys = (wl.k_idx[sl].clone(), wl.k_scale[sl].clone(), wl.kv[sl].clone())
    part = shard.ShardForward(dsa, pb, rb, n, wl.q_idx[sl], wl.q_scale[sl], wl.w[sl], wl.q[sl])
    del wl
    torch.cuda.empty_cache()

    def step():
        with torch.cuda.stream(stream):
            keys = shard.gather_keys(*local_keys, ranges)
        dsa.check(part(*keys, stream=stream), "sharded prefill")
        return keys

    steps = max(1, min(args.steps, args.prefill_steps))
    for _ in range(max(1, min(args.warmup, 3))):
        step()
    torch.cuda.synchronize()
    torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    torch.distributed.barrier()
    ms_step = max_over_ranks(e0.elapsed_time(e1), world, dev) / steps
    st, _ = dsa.dsa_read_device_status(part.status, stream)
    dsa.check(st, "sharded prefill status")
    seqlens = make_config_seqlens(cfg)
    T = sum(seqlens)
    from dsa_workloads import FULL
    f8, f16 = prefill_flops(seqlens, FULL)
    p8 = 2.0 * peaks["bf16_sustained"]
    ideal_ms = (f8 / (p8 * 1e12) + f16 / (peaks["bf16_sustained"] * 1e12)) * 1e3 / world
    res = {"workload": CONFIGS[cfg]["name"], "value": round(T / (ms_step / 1e3), 1),
           "unit": "tokens/s", "ms_per_step": round(ms_step, 3), "steps": steps,
           "scaling": "strong", "ranges": ranges,
           "roofline": {"bound": "tensor", "frac": round(ideal_ms / ms_step, 4),
                        "ideal_ms_per_gpu": round(ideal_ms, 3)},
           "note": "one problem split over the ranks by query rows; each step all-gathers the "
                   "key-side rows (NCCL) and runs dsa_forward_rows on the rank's rows"}
    del part, local_keys
    torch.cuda.empty_cache()
    return res


def make_config_seqlens(cfg):
    from dsa_workloads import CONFIGS
    return list(CONFIGS[cfg]["seqlens"])


def run_prefill(args, dsa, dev, stream, peaks, rank, world, cfg):
    if world > 1:
        return run_prefill_sharded(args, dsa, dev, stream, peaks, rank, world, cfg)
    from dsa_workloads import make_config, CONFIGS, sample_rows
    wl = make_config(cfg, device=dev, seed=rank_seed(cfg, rank))
    fwd = dsa.Forward(wl, keep_idx=False)
    steps = max(1, min(args.steps, args.prefill_steps))
    for _ in range(max(1, min(args.warmup, 3))):
        dsa.check(fwd(stream), "prefill forward")
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        dsa.check(fwd(stream), "prefill forward")
    e1.record(stream)
    torch.cuda.synchronize()
    ms_step = max_over_ranks(e0.elapsed_time(e1), world, dev) / steps
    st, raw = dsa.dsa_read_device_status(fwd.status, stream)
    dsa.check(st, "prefill device status")
    del fwd
    sm = torch.cuda.get_device_properties(dev).multi_processor_count
    split, n_launch = prefill_stage_split(dsa, wl, stream, sm)
    f8, f16 = prefill_flops(wl.seqlens, wl.dims)
    p8 = 2.0 * peaks["bf16_sustained"]
    ideal_ms = (f8 / (p8 * 1e12) + f16 / (peaks["bf16_sustained"] * 1e12)) * 1e3
    T = wl.total_rows
    stage_sum = sum(split.values())
    res = {"workload": CONFIGS[cfg]["name"], "value": round(weak_value(world, T, ms_step), 1),
           "unit": "tokens/s", "ms_per_step": round(ms_step, 3), "steps": steps,
           "roofline": {"bound": "tensor", "frac": round(ideal_ms / ms_step, 4),
                        "ideal_ms": round(ideal_ms, 3), "flops_fp8": f8, "flops_bf16": f16,
                        "peak_bf16_tflops": peaks["bf16_sustained"],
                        "peak_fp8_tflops": p8,
                        "peak_note": "bf16 sustained measured; fp8 = 2x bf16 (nominal ratio)"},
           "kernel_ms": {k: round(v, 3) for k, v in sorted(split.items())},
           "kernel_share": {k: round(v / stage_sum, 4) for k, v in sorted(split.items())},
           "kernel_ms_note": "one pass of the same chunks through the stage calls, CUDA events "
                             "around every launch; summed per stage (the forward runs them "
                             "back to back, so the sum is a little above ms_per_step)",
           "gpu_launches_per_step": n_launch}
    if rank == 0 and not args.no_cpu:
        import oracle
        rows = sample_rows(wl, 2)
        t0 = time.perf_counter()
        oracle.forward_rows(wl, rows)
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": round(len(rows) / dt, 3), "unit": "tokens/s",
                               "cores": oracle.num_threads(), "kind": "oracle",
                               "sample": f"{len(rows)} sampled rows (2 per sequence; indexer over "
                                         f"every prior key, top-k, fp64 attention), {dt:.1f} s"}
    del wl
    torch.cuda.empty_cache()
    return res


def run_indexer_train(args, dsa, dev, stream, peaks, rank, world, cpu_leg):
    """One training step of the indexer (sparse stage) on prefill_L16k: the KL target from the
    main attention and the KL loss with its gradients (both on the tensor cores),
    after one forward pass that keeps the selection, the selected keys' scores and the LSE.  dk is zeroed inside the
    step (the backward adds into it)."""
    from dsa_workloads import make_config, make_prefill, CONFIGS, FULL
    if args.train_len == CONFIGS[TRAIN_CFG]["seqlens"][0]:
        wl = make_config(TRAIN_CFG, device=dev, seed=rank_seed(TRAIN_CFG, rank))
        name = CONFIGS[TRAIN_CFG]["name"]
    else:   # profiling only: a shorter sequence of the same kind
        c = CONFIGS[TRAIN_CFG]
        name = f"prefill_L{args.train_len}"
        wl = make_prefill(TRAIN_CFG, [args.train_len], FULL, c["needles"], dev,
                          seed=rank_seed(TRAIN_CFG, rank), name=name)
    d = wl.dims
    T, K = wl.total_rows, d["topk"]
    fwd = dsa.Forward(wl, keep_idx=True, keep_sel=True)
    dsa.check(fwd(stream), "forward for the training step")
    pb = fwd.pb
    target = torch.empty(T, K, dtype=torch.float32, device=dev)
    loss = torch.empty(T, dtype=torch.float32, device=dev)
    dw = torch.empty(T, d["h_idx"], dtype=torch.float32, device=dev)
    dq = torch.empty(T, d["h_idx"], d["d_idx"], dtype=torch.float32, device=dev)
    dk = torch.empty(wl.k_idx.shape[0], d["d_idx"], dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        dsa.check(dsa.dsa_indexer_kl_target(pb, wl.q, wl.kv, fwd.idx, fwd.lse, 0, T, target,
                                            status, stream), "kl target")
        if ev is not None:
            ev[1].record(stream)
        with torch.cuda.stream(stream):
            dk.zero_()
        dsa.check(dsa.dsa_indexer_kl_backward(pb, wl.q_idx, wl.q_scale, wl.w, wl.k_idx,
                                              wl.k_scale, fwd.idx, target, 0, T, loss, dw, dq,
                                              dk, status, stream, sel=fwd.sel), "kl backward")
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, args.prefill_steps))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        step(evs[i])
    e1.record(stream)
    torch.cuda.synchronize()
    ms_step = max_over_ranks(e0.elapsed_time(e1), world, dev) / steps
    t_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / steps
    b_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / steps
    st, _ = dsa.dsa_read_device_status(status, stream)
    dsa.check(st, "training step status")
    f_t, f_b = train_flops(wl.seqlens, d)
    t_tf = f_t / (t_ms / 1e3) / 1e12
    res = {"workload": name, "value": round(weak_value(world, T, ms_step), 1),
           "unit": "tokens/s", "ms_per_step": round(ms_step, 3), "steps": steps,
           "kernel_ms": {"kl_target": round(t_ms, 3), "kl_backward": round(b_ms, 3)},
           "roofline": kl_backward_roofline(f_b, b_ms, peaks["bf16_sustained"]),
           "target_roofline": {"kernel": "dsa_sparse_mla_kernel (target mode)",
                               "bound": "tensor", "achieved": round(t_tf, 1),
                               "peak": peaks["bf16_sustained"], "unit": "TFLOP/s",
                               "frac": round(t_tf / peaks["bf16_sustained"], 4), "flops": f_t},
           "gpu_launches_per_step": 2,
           "note": "after one forward that keeps the selection, its scores and the LSE; per "
                   "step: target, dk zeroed (a torch memset), backward (softmax over the kept "
                   "scores)"}
    if cpu_leg:
        import oracle
        rows = [int(x) for x in np.linspace(T // 2, T - 1, 16)]
        t0 = time.perf_counter()
        sc = oracle.indexer_rows(wl, rows)
        sel = oracle.topk_rows([sc[r] for r in rows], K)
        tg = oracle.kl_target_rows(wl, rows, sel)
        oracle.indexer_kl_rows(wl, rows, sel, tg)
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": round(len(rows) / dt, 3), "unit": "tokens/s",
                               "cores": oracle.num_threads(), "kind": "oracle",
                               "sample": f"{len(rows)} rows of the second half (indexer, top-k, "
                                         f"target, loss and gradients per row), {dt:.1f} s"}
    del fwd, target, dq, dk
    torch.cuda.empty_cache()
    return res


def time_cache_append(args, dsa, wl, stream, peaks, cpu_leg):
    """The decode cache append (one new token per sequence quantised into the paged caches),
    timed on its own after the decode step's numbers were taken: it rewrites each sequence's
    last cache row.  Launch-bound by nature (189 KB at B = 64); reported beside the oracle doing
    the same work per token on the host."""
    import oracle
    pb = dsa.problem_of(wl)
    B, d = wl.batch, wl.dims
    g = torch.Generator(device=wl.kv.device).manual_seed(77)
    k_new = torch.randn(B, d["d_idx"], generator=g, device=wl.kv.device)
    kv_new = torch.randn(B, d["d_qk"], generator=g, device=wl.kv.device).to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device=wl.kv.device)

    def call():
        dsa.check(dsa.dsa_cache_append(pb, k_new, kv_new, wl.k_idx, wl.k_scale, wl.kv, status,
                                       stream), "cache_append")
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(20, args.steps)
    e0.record(stream)
    for _ in range(n):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / n
    st, _ = dsa.dsa_read_device_status(status, stream)
    dsa.check(st, "cache_append status")
    per_tok = 4 * d["d_idx"] + 2 * d["d_qk"] + d["d_idx"] + 4 + 2 * d["d_qk"]
    gbs = B * per_tok / (us / 1e6) / 1e9
    res = {"us_per_call": round(us, 2), "batch": B, "bytes_per_call": B * per_tok,
           "achieved_gbs": round(gbs, 1), "peak_gbs": peaks["hbm"],
           "frac": round(gbs / peaks["hbm"], 5), "gpu_launches_per_call": 1,
           "note": "one warp per sequence; launch latency, not bandwidth, sets the time"}
    if cpu_leg:
        # CPU baseline: the oracle doing the same work per token (quantise the keys, write the
        # three rows into host caches)
        import oracle
        kn, kvn = k_new.cpu().numpy(), kv_new.view(torch.int16).cpu().numpy()
        z8 = np.zeros((B, d["d_idx"]), np.uint8)
        zs = np.zeros(B, np.float32)
        z16 = np.zeros((B, d["d_qk"]), np.int16)
        reps = 20
        t0 = time.perf_counter()
        for _ in range(reps):
            codes, scales = oracle.quantize_e4m3(kn)
            z8[:] = codes
            zs[:] = scales
            z16[:] = kvn
        res["cpu_baseline"] = {"us_per_call": round((time.perf_counter() - t0) / reps * 1e6, 1),
                               "kind": "oracle", "cores": 1,
                               "sample": f"the same {B} tokens, host caches"}
    return res


def probe_dsmem(dsa, dev, stream, nbytes=32 * 1024, reps=256):
    """Distributed-shared-memory exchange rate between the two CTAs (two SMs) of a cluster, both
    directions at once: one cluster alone and one per SM pair; per SM = bytes it sends / time."""
    sm = torch.cuda.get_device_properties(dev).multi_processor_count
    res = {"bytes_per_round": nbytes, "rounds": reps}
    for name, clusters in (("one_pair", 1), ("all_pairs", sm // 2)):
        ns = torch.zeros(clusters, dtype=torch.int64, device=dev)
        bad = torch.zeros(1, dtype=torch.int32, device=dev)
        for _ in range(2):   # the first launch warms up
            dsa.check(dsa.dsa_probe_dsmem(clusters, nbytes, reps, ns, bad, stream), "dsmem probe")
        torch.cuda.synchronize()
        dsa.check(0 if int(bad.item()) == 0 else dsa.DSA_ERR_CUDA, "dsmem probe words")
        t = ns.double().mean().item()
        res[name] = {"clusters": clusters, "gbs_per_sm": round(nbytes * reps / t, 2),
                     "gbs_total": round(2 * clusters * nbytes * reps / t, 1)}
    return res


def probe_page_stream(dsa, wl, dev, stream, roof, reps=5):
    """Read rate of the decode indexer's key pages (each 64-row page with its 64 scales, in
    block-table order) with the indexer producer's copies and no arithmetic: the practical
    ceiling of the indexer's stream on this access pattern, with 1 to 8 CTAs per SM (fewer
    pages in flight per CTA as they grow); the indexer's own rate is reported as a fraction of
    the best.  The 1.1 GB of pages exceed L2, so no flush is needed."""
    if wl.block_table is None or wl.k_scale is not None:
        return None
    nb = [(L + 63) // 64 for L in wl.seqlens]
    ids = torch.cat([wl.block_table[b, :n] for b, n in enumerate(nb)]).contiguous()
    bb = int(wl.k_idx.shape[1])
    nbytes = ids.numel() * bb
    res = {"blocks": ids.numel(), "block_bytes": bb}
    bad = torch.zeros(1, dtype=torch.int32, device=dev)
    best = 0.0

    def launch(cps):
        dsa.check(dsa.dsa_probe_page_stream(wl.k_idx, ids, int(wl.k_idx.shape[0]),
                                            wl.dims["d_idx"], cps, bad, stream),
                  "page stream probe")

    for cps in (1, 2, 3, 4, 6, 8):
        for _ in range(2):                       # warm-up
            launch(cps)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            launch(cps)
        e1.record(stream)
        torch.cuda.synchronize()
        gbs = nbytes * reps / (e0.elapsed_time(e1) * 1e-3) / 1e9
        res[f"gbs_ctas_per_sm_{cps}"] = round(gbs, 1)
        best = max(best, gbs)
    dsa.check(0 if int(bad.item()) == 0 else dsa.DSA_ERR_CUDA, "page stream probe ids")
    res["gbs"] = round(best, 1)
    res["indexer_frac_of_stream"] = round(roof["achieved"] / best, 4)
    return res


def load_traffic(name):
    """DRAM bytes per launch from the committed ncu summary, or None when the kernel source has
    changed since the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(name)
    if rec is None:
        return None
    src = os.path.join(ROOT, "sparse_attention_long_04_b200", "csrc", "indexer.cuh")
    with open(src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()[:16]
    return rec["bytes_per_launch"] if h == rec.get("indexer_cuh_sha256_16") else None


# ------------------------------------------------------------------------------ CPU oracle

def oracle_sample(wl, n_rows):
    """A decode workload holding only `n_rows` sequences of `wl`, laid out contiguously on the
    host (a gather of the inputs; no arithmetic), for timing the oracle."""
    import oracle
    from dsa_workloads import Workload
    rows = list(range(n_rows))
    L = wl.max_seqlen
    bt = wl.block_table[:n_rows].long()
    phys = (bt[:, torch.arange(L, device=bt.device) // 64] * 64 +
            torch.arange(L, device=bt.device) % 64).reshape(-1)
    codes, scales = oracle.key_rows(wl, phys.cpu().numpy())
    return Workload(cfg_id=wl.cfg_id, name=wl.name, mode="decode", dims=wl.dims,
                    softmax_scale=wl.softmax_scale, seqlens=wl.seqlens[:n_rows],
                    q_idx=wl.q_idx[rows].cpu(), q_scale=wl.q_scale[rows].cpu(),
                    w=wl.w[rows].cpu(), k_idx=torch.from_numpy(codes),
                    k_scale=torch.from_numpy(scales), q=wl.q[rows].cpu(), kv=wl.kv[phys].cpu(),
                    seq_lens=wl.seq_lens[:n_rows].cpu(), block_table=None, max_seqlen=L)


def cpu_baseline(wl, budget_s=15.0):
    import oracle
    threads = oracle.num_threads()
    n = max(1, min(wl.batch, threads))
    sub = oracle_sample(wl, n)
    t0 = time.perf_counter()
    oracle.forward_rows(sub, list(range(n)))
    dt = time.perf_counter() - t0
    if dt < budget_s / 3 and n < wl.batch:          # grow the sample toward the budget
        n2 = min(wl.batch, max(n + 1, int(n * budget_s / 2 / max(dt, 1e-3))))
        sub = oracle_sample(wl, n2)
        t0 = time.perf_counter()
        oracle.forward_rows(sub, list(range(n2)))
        dt = time.perf_counter() - t0
        n = n2
    return {"value": round(n / dt, 4), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} of {wl.batch} decode rows of {wl.name} (full 131072-key indexer, "
                      f"top-k, fp64 attention per row), {dt:.1f} s"}


def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores, on the decode workload's metric."""
    if rank != 0:
        return None
    from dsa_workloads import make_config, CONFIGS
    import oracle
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    wl = make_config(DECODE_CFG, device=dev)
    threads = oracle.num_threads()
    n = max(1, min(wl.batch, threads))
    sub = oracle_sample(wl, n)
    for _ in range(args.warmup):
        oracle.forward_rows(sub, [0])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward_rows(sub, list(range(n)))
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": CONFIGS[DECODE_CFG]["name"], "batch": wl.batch,
                       "context": wl.max_seqlen, "parallelism": "replicas1"},
            "cpu_baseline": {"value": round(value, 4), "kind": "oracle", "cores": threads,
                             "sample": f"{n} decode rows per step of {wl.name}"},
            "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def spawn_ranks(n: int) -> int:
    """`--gpus N` without a launcher: start N ranks of this script on this node (one per GPU)
    through torch.distributed.run, with the same arguments; rank 0 prints the line.  Never
    reports a one-GPU number for N > 1."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the secondary full-shape workloads (decode_B32_N32k, prefill_L16k)")
    ap.add_argument("--no-train", action="store_true",
                    help="skip the indexer training step (prefill_L16k)")
    ap.add_argument("--train-only", action="store_true",
                    help="profiling only: time just the indexer training step")
    ap.add_argument("--train-len", type=int, default=16384,
                    help="profiling only: sequence length of the training step")
    ap.add_argument("--prefill-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--prefill-only", type=int, default=0, choices=[0, 1, 4, 5],
                    help="profiling only: time just the prefill of this workload (4 or 5)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="profiling only: decode sequences (default: the workload's 64)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}: one rank per GPU")
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        if args.prefill_only:
            import sparse_attention_long_04_b200 as dsa
            global PREFILL_CFG
            PREFILL_CFG = args.prefill_only
            dev = torch.device("cuda", local_rank)
            torch.cuda.set_device(dev)
            line = run_prefill(args, dsa, dev, torch.cuda.current_stream(), read_peaks(), rank,
                               world, PREFILL_CFG)
            if rank == 0:
                print(json.dumps(line), flush=True)
            return
        if args.train_only:
            import sparse_attention_long_04_b200 as dsa
            dev = torch.device("cuda", local_rank)
            torch.cuda.set_device(dev)
            line = run_indexer_train(args, dsa, dev, torch.cuda.current_stream(), read_peaks(),
                                     rank, world, cpu_leg=rank == 0 and not args.no_cpu)
            if rank == 0:
                print(json.dumps(line), flush=True)
            return
        line = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
