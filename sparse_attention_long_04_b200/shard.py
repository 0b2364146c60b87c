"""Prefill across GPUs, one process per GPU: each rank takes a contiguous range of query rows.

Every query row attends to the prior keys of its whole sequence, so the ranks first exchange the
key-side rows (the e4m3 indexer key with its scale, 132 B per token at full shapes, and the
576-d latent row, 1152 B) with one all-gather each, into local memory; then each rank runs the
whole path on its own rows with dsa_forward_rows.  Top-k and attention need nothing else from
the other ranks.  This is the split of the pages' long-context prefill ("Costs vs. position
(128k)", "DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek Sparse Attention (DSA)") over
several GPUs; the pages themselves describe no multi-GPU layout.

Only plumbing lives here: the row split (host arithmetic on lengths), the all-gathers
(torch.distributed: NCCL between GPUs, gloo on CPU) and the call into the library.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch


def row_costs(seqlens: Sequence[int], dims: dict) -> List[Tuple[int, int, int]]:
    """Per sequence (first packed row, length, topk): the pieces split_rows weighs."""
    out, off = [], 0
    for L in seqlens:
        out.append((off, int(L), int(dims["topk"])))
        off += int(L)
    return out


def _prefix_cost(L: int, K: int, n: int, a: float, b: float) -> float:
    """Cost of a sequence's first n rows: row p scores p + 1 keys (a per key) and attends to
    min(p + 1, K) of them (b per key)."""
    n = max(0, min(n, L))
    dense = min(n, K)
    return a * n * (n + 1) / 2 + b * (dense * (dense + 1) / 2 + (n - dense) * K)


def split_rows(seqlens: Sequence[int], dims: dict, world: int) -> List[Tuple[int, int]]:
    """Contiguous query-row ranges (row_begin, row_count), one per rank, that cover every packed
    row once and balance the work: the indexer's 2 H_I D_I FLOP per (row, prior key) in e4m3
    (counted at half the bf16 cost) and the attention's 2 H (D_qk + D_v) FLOP per (row, selected
    key) in bf16.  Ranks may get empty ranges when there are fewer rows than ranks."""
    a = dims["h_idx"] * dims["d_idx"]                 # 2 H_I D_I / 2 (e4m3 at twice the rate)
    b = 2 * dims["h"] * (dims["d_qk"] + dims["d_v"])
    seqs = row_costs(seqlens, dims)
    total_rows = sum(int(L) for L in seqlens)
    totals = [_prefix_cost(L, K, L, a, b) for _, L, K in seqs]
    grand = sum(totals)

    def cost_before(row: int) -> float:               # work of packed rows [0, row)
        c = 0.0
        for (off, L, K), t in zip(seqs, totals):
            if row >= off + L:
                c += t
            elif row > off:
                c += _prefix_cost(L, K, row - off, a, b)
        return c

    cuts = [0]
    for r in range(1, world):
        target = grand * r / world
        lo, hi = cuts[-1], total_rows                 # first row with cost_before >= target
        while lo < hi:
            mid = (lo + hi) // 2
            if cost_before(mid) < target:
                lo = mid + 1
            else:
                hi = mid
        cuts.append(lo)
    cuts.append(total_rows)
    return [(cuts[i], cuts[i + 1] - cuts[i]) for i in range(world)]


def all_gather_rows(local: torch.Tensor, ranges: Sequence[Tuple[int, int]], group=None
                    ) -> torch.Tensor:
    """Rows [row_begin, row_begin + row_count) of a tensor from every rank, concatenated in rank
    order (= packed row order): each rank passes its own rows; the result holds all of them.
    One all-gather of equal-size pieces (padded to the longest range)."""
    import torch.distributed as dist
    world = len(ranges)
    longest = max(n for _, n in ranges)
    width = local.element_size()
    for x in local.shape[1:]:
        width *= int(x)
    flat = local.contiguous().view(torch.uint8).reshape(local.shape[0], width)
    piece = torch.zeros(longest, width, dtype=torch.uint8, device=local.device)
    piece[: flat.shape[0]] = flat
    gathered = torch.empty(world * longest, width, dtype=torch.uint8, device=local.device)
    dist.all_gather_into_tensor(gathered, piece, group=group)
    rows = [gathered[r * longest: r * longest + n] for r, (_, n) in enumerate(ranges)]
    full = torch.cat(rows, 0).contiguous()
    return full.view(local.dtype).reshape((-1,) + tuple(local.shape[1:]))


def gather_keys(k_idx: torch.Tensor, k_scale: torch.Tensor, kv: torch.Tensor,
                ranges: Sequence[Tuple[int, int]], group=None):
    """The key-side rows of every rank (e4m3 indexer keys, their scales, latent rows)."""
    return (all_gather_rows(k_idx, ranges, group), all_gather_rows(k_scale, ranges, group),
            all_gather_rows(kv, ranges, group))


class ShardForward:
    """One rank's part of a sharded prefill: its query rows (local arrays), the gathered keys,
    and the outputs of its rows; calling it runs dsa_forward_rows on the rank's range."""

    def __init__(self, dsa, pb, row_begin: int, row_count: int, q_idx, q_scale, w, q,
                 keep_idx: bool = False):
        d = pb.dims
        dev = q.device
        self.dsa, self.pb = dsa, pb
        self.row_begin, self.row_count = row_begin, row_count
        self.q_idx, self.q_scale, self.w, self.q = q_idx, q_scale, w, q
        self.ws_bytes = dsa.dsa_forward_workspace_size(pb)
        self.ws = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device=dev)
        self.out = torch.empty(row_count, d.h, d.d_v, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(row_count, d.h, dtype=torch.float32, device=dev)
        self.idx = (torch.empty(row_count, d.topk, dtype=torch.int32, device=dev)
                    if keep_idx else None)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def __call__(self, k_idx, k_scale, kv, stream=None) -> int:
        if self.row_count == 0:
            return self.dsa.DSA_OK
        return self.dsa.dsa_forward_rows(self.pb, self.row_begin, self.row_count, self.q_idx,
                                         self.q_scale, self.w, k_idx, k_scale, self.q, kv,
                                         self.idx, self.out, self.lse, self.ws, self.ws_bytes,
                                         self.status, stream)
