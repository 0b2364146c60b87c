"""Seeded synthetic workloads for the DSA hot path (lightning indexer -> top-k -> sparse MLA-MQA).

This module only *draws* inputs.  It holds none of the method's arithmetic: it samples
Gaussian / uniform tensors, plants "needle" keys, quantises the indexer tensors to FP8 e4m3
with a per-token fp32 scale (the input format the indexer consumes, "FP8 index" in
"DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek Sparse Attention (DSA)", pipeline
summary), and builds the sequence metadata (cu_seqlens, seq_lens, block tables).  Both the
CPU oracle and the CUDA path consume the exact bytes produced here.

Workload shapes follow the five DSA workloads this repository is measured on:

  tiny_prefill_L1024         1 causal sequence of 1024 tokens, indexer 4x32, top-k 64,
                             16 heads, latent 128+32, values 128, 8 needles per 128-row band
  decode_B32_N32k            32 sequences x 32768 context, full shapes, 1 % boosted keys
  decode_B64_N128k_paged     64 x 131072 context, 64-token pages, random block table,
                             0.5 % planted keys; each page of the indexer cache holds its 64
                             key rows followed by their 64 scales
  prefill_L16k               1 causal sequence of 16384 tokens, needles
  prefill_varlen_T276480     8 packed sequences {4096, 8192, 16384, 16384, 32768, 65536,
                             131072, 2048}

Full shapes: indexer 64 heads x 128 dims (e4m3), top-k 2048, 128 query heads, latent KV
512 + 64 RoPE = 576 bf16, value dim 512 (the first 512 latent dims).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import torch

E4M3_MAX = 448.0
BLOCK_SIZE = 64

FULL = dict(h_idx=64, d_idx=128, topk=2048, h=128, d_qk=576, d_v=512)
TINY = dict(h_idx=4, d_idx=32, topk=64, h=16, d_qk=160, d_v=128)

# name -> description.  "needles": per 128-row query band, count of planted keys with a
# +3 sigma indexer similarity.  "boost": fraction of decode context keys moved +2 sigma
# toward the query.
CONFIGS: Dict[int, dict] = {
    1: dict(name="tiny_prefill_L1024", mode="prefill", seqlens=[1024], needles=8, **TINY),
    2: dict(name="decode_B32_N32k", mode="decode", batch=32, ctx=32768, paged=False,
            boost=0.01, **FULL),
    3: dict(name="decode_B64_N128k_paged", mode="decode", batch=64, ctx=131072, paged=True,
            boost=0.005, scale_layout="interleaved", **FULL),
    4: dict(name="prefill_L16k", mode="prefill", seqlens=[16384], needles=8, **FULL),
    5: dict(name="prefill_varlen_T276480", mode="prefill",
            seqlens=[4096, 8192, 16384, 16384, 32768, 65536, 131072, 2048], needles=8, **FULL),
}


@dataclass
class Workload:
    """One batch of DSA inputs.  All tensors live on ``device``.

    Layouts (row-major, contiguous):
      q_idx      uint8 [T, h_idx, d_idx]   e4m3 bytes of the indexer queries
      q_scale    f32   [T, h_idx]          per-(token, indexer head) dequant scale
      w          f32   [T, h_idx]          indexer head weights
      k_idx      uint8 [R, d_idx]          e4m3 bytes of the indexer keys (R physical rows), or
                                           with interleaved scales uint8 [R/64, 64*(d_idx+4)]:
                                           each 64-row block's key rows, then its 64 fp32 scales
      k_scale    f32   [R] or None         per-key dequant scale (None: inside k_idx's blocks)
      q          bf16  [T, h, d_qk]        absorbed MLA queries
      kv         bf16  [R, d_qk]           latent KV rows (values = first d_v dims)
    Prefill: T = R = total packed tokens; row r of sequence b sits at cu_seqlens[b] + pos.
    Decode : T = batch (one new token per sequence, position seq_lens[b]-1); physical row
             of logical key s of sequence b is block_table[b, s // 64] * 64 + s % 64 when
             paged, else b * max_seqlen + s.
    """
    cfg_id: int
    name: str
    mode: str
    dims: dict
    softmax_scale: float
    seqlens: List[int]
    q_idx: torch.Tensor
    q_scale: torch.Tensor
    w: torch.Tensor
    k_idx: torch.Tensor
    k_scale: Optional[torch.Tensor]
    q: torch.Tensor
    kv: torch.Tensor
    cu_seqlens: Optional[torch.Tensor] = None     # int32 [batch+1] (prefill)
    seq_lens: Optional[torch.Tensor] = None       # int32 [batch]   (decode)
    block_table: Optional[torch.Tensor] = None    # int32 [batch, max_blocks] (paged decode)
    max_seqlen: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return len(self.seqlens)

    @property
    def total_rows(self) -> int:
        return self.q.shape[0]

    def to(self, device) -> "Workload":
        out = Workload(**{k: getattr(self, k) for k in self.__dataclass_fields__})
        for k in ("q_idx", "q_scale", "w", "k_idx", "k_scale", "q", "kv", "cu_seqlens",
                  "seq_lens", "block_table"):
            v = getattr(self, k)
            if v is not None:
                setattr(out, k, v.to(device))
        return out


def _gen(seed: int, tensor_id: int, seq_id: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + tensor_id * 7919 + seq_id * 104_729) & ((1 << 62) - 1))
    return g


def quantize_e4m3_rows(x: torch.Tensor, group_dims: int):
    """Per-row e4m3 quantisation over the last ``group_dims`` dims: scale = amax / 448
    (amax = 0 -> scale 1), bytes = round-to-nearest-even cast of x / scale.  Returns
    (uint8 bytes with x's shape, fp32 scale with the leading shape)."""
    lead = x.shape[: x.dim() - group_dims]
    flat = x.reshape(*lead, -1).float()
    amax = flat.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (flat / scale.unsqueeze(-1)).clamp_(-E4M3_MAX, E4M3_MAX)
    q8 = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(x.shape)
    return q8.contiguous(), scale.float().contiguous()


def interleave_key_blocks(k8: torch.Tensor, ks: torch.Tensor, block: int = BLOCK_SIZE):
    """The paged indexer cache with each block's scales stored right after its key rows:
    uint8 [R / block, block * d + block * 4] (a layout change only; the bytes are the same)."""
    R, d = k8.shape
    nb = R // block
    keys = k8.reshape(nb, block * d)
    sc = ks.contiguous().view(torch.uint8).reshape(nb, block * 4)
    return torch.cat([keys, sc], dim=1).contiguous()


def _unit(v: torch.Tensor) -> torch.Tensor:
    return v / v.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_prefill(cfg_id: int, seqlens: List[int], dims: dict, needles: int, device,
                 seed: Optional[int] = None, name: Optional[str] = None,
                 softmax_scale: Optional[float] = None, band: int = 128) -> Workload:
    """Packed varlen causal prefill.  Each sequence draws from its own seeded sub-streams.

    Needles: each band of ``band`` consecutive query positions gets a seeded unit vector u;
    the band's indexer queries get q_I += u (every indexer head) and ``needles`` seeded key
    positions before the band's end get k_I += 3 sqrt(d_idx) u, a +3 sigma shift of q.k for
    N(0,1) entries.  Latent KV and MLA queries stay pure N(0,1)."""
    seed = 1000 + cfg_id if seed is None else seed
    h_idx, d_idx, h, d_qk = dims["h_idx"], dims["d_idx"], dims["h"], dims["d_qk"]
    T = int(sum(seqlens))
    q8 = torch.empty(T, h_idx, d_idx, dtype=torch.uint8, device=device)
    qs = torch.empty(T, h_idx, dtype=torch.float32, device=device)
    k8 = torch.empty(T, d_idx, dtype=torch.uint8, device=device)
    ks = torch.empty(T, dtype=torch.float32, device=device)
    w = torch.empty(T, h_idx, dtype=torch.float32, device=device)
    q = torch.empty(T, h, d_qk, dtype=torch.bfloat16, device=device)
    kv = torch.empty(T, d_qk, dtype=torch.bfloat16, device=device)
    off = 0
    for b, L in enumerate(seqlens):
        sl = slice(off, off + L)
        qi = torch.randn(L, h_idx, d_idx, generator=_gen(seed, 1, b, device), device=device)
        ki = torch.randn(L, d_idx, generator=_gen(seed, 2, b, device), device=device)
        if needles > 0 and L > 0:
            nb = (L + band - 1) // band
            g = _gen(seed, 3, b, device)
            u = _unit(torch.randn(nb, d_idx, generator=g, device=device))
            band_of_row = torch.arange(L, device=device) // band
            qi += u[band_of_row].unsqueeze(1)
            band_end = torch.clamp((torch.arange(nb, device=device) + 1) * band, max=L)
            pos = (torch.rand(nb, needles, generator=g, device=device)
                   * band_end.unsqueeze(1).float()).long().clamp_(max=L - 1)
            ki.index_add_(0, pos.reshape(-1),
                          (3.0 * math.sqrt(d_idx)) * u.repeat_interleave(needles, dim=0))
        # literal per-token q scale: one amax over the token's h_idx x d_idx values, stored per
        # indexer head
        q8[sl], s_tok = quantize_e4m3_rows(qi, 2)
        qs[sl] = s_tok.unsqueeze(1)
        k8[sl], ks[sl] = quantize_e4m3_rows(ki, 1)
        del qi, ki
        w[sl] = torch.rand(L, h_idx, generator=_gen(seed, 4, b, device), device=device)
        gq, gkv = _gen(seed, 5, b, device), _gen(seed, 6, b, device)
        step = max(1, (1 << 26) // (h * d_qk))          # bounded fp32 temporaries
        for r0 in range(0, L, step):
            r1 = min(L, r0 + step)
            q[off + r0:off + r1] = torch.randn(r1 - r0, h, d_qk, generator=gq, device=device)
        step = max(1, (1 << 26) // d_qk)
        for r0 in range(0, L, step):
            r1 = min(L, r0 + step)
            kv[off + r0:off + r1] = torch.randn(r1 - r0, d_qk, generator=gkv, device=device)
        off += L
    cu = torch.tensor([0] + list(torch.tensor(seqlens).cumsum(0).tolist()), dtype=torch.int32,
                      device=device)
    return Workload(cfg_id=cfg_id, name=name or f"prefill_{len(seqlens)}seq", mode="prefill",
                    dims=dict(dims), softmax_scale=softmax_scale or 1.0 / math.sqrt(d_qk),
                    seqlens=list(seqlens), q_idx=q8, q_scale=qs, w=w, k_idx=k8, k_scale=ks,
                    q=q, kv=kv, cu_seqlens=cu, max_seqlen=max(seqlens))


def make_decode(cfg_id: int, batch: int, ctx, dims: dict, boost: float, paged: bool, device,
                seed: Optional[int] = None, name: Optional[str] = None,
                softmax_scale: Optional[float] = None, total_blocks: Optional[int] = None,
                scale_layout: str = "separate") -> Workload:
    """Decode: one new token per sequence, whose k_I and latent KV are already in the cache
    (query position = seq_len - 1).  ``ctx`` is an int or a per-sequence list.

    Boost: u_b = unit(sum_j w_j q_I[b, j]); a seeded fraction ``boost`` of the context
    positions get k_I += 2 sqrt(d_idx) u_b.  Paged: 64-token blocks, the block table is a
    seeded permutation of the physical blocks.  scale_layout "interleaved" (paged only) stores
    each block's 64 key scales right after its 64 key rows (k_scale None)."""
    seed = 1000 + cfg_id if seed is None else seed
    h_idx, d_idx, h, d_qk = dims["h_idx"], dims["d_idx"], dims["h"], dims["d_qk"]
    lens = [int(ctx)] * batch if isinstance(ctx, int) else [int(c) for c in ctx]
    assert len(lens) == batch and min(lens) >= 1
    max_len = max(lens)
    max_blocks = (max_len + BLOCK_SIZE - 1) // BLOCK_SIZE
    if paged:
        nblk = total_blocks or batch * max_blocks
        assert nblk >= batch * max_blocks
        perm = torch.randperm(nblk, generator=_gen(seed, 7, 0, device), device=device)
        block_table = perm[: batch * max_blocks].view(batch, max_blocks).to(torch.int32)
        rows = nblk * BLOCK_SIZE
    else:
        block_table = None
        rows = batch * max_len
    qi = torch.randn(batch, h_idx, d_idx, generator=_gen(seed, 1, 0, device), device=device)
    w = torch.rand(batch, h_idx, generator=_gen(seed, 4, 0, device), device=device)
    ki = torch.randn(rows, d_idx, generator=_gen(seed, 2, 0, device), device=device)
    if boost > 0:
        u = _unit((w.unsqueeze(-1) * qi).sum(1))                     # [batch, d_idx]
        g = _gen(seed, 3, 0, device)
        for b in range(batch):
            n_pick = max(1, int(round(boost * lens[b])))
            s = torch.randperm(lens[b], generator=g, device=device)[:n_pick]
            if paged:
                phys = block_table[b, s // BLOCK_SIZE].long() * BLOCK_SIZE + s % BLOCK_SIZE
            else:
                phys = b * max_len + s
            ki[phys] += (2.0 * math.sqrt(d_idx)) * u[b]
    q8, qs = quantize_e4m3_rows(qi, 2)
    qs = qs.unsqueeze(1).expand(-1, h_idx).contiguous()
    k8, ks = quantize_e4m3_rows(ki, 1)
    del ki
    if scale_layout == "interleaved":
        assert paged, "interleaved scales need the paged layout"
        k8, ks = interleave_key_blocks(k8, ks), None
    q = torch.randn(batch, h, d_qk, generator=_gen(seed, 5, 0, device), device=device
                    ).to(torch.bfloat16)
    kv = torch.empty(rows, d_qk, dtype=torch.bfloat16, device=device)
    step = 1 << 24
    g6 = _gen(seed, 6, 0, device)
    for r0 in range(0, rows, step // d_qk):       # bounded fp32 temporaries
        r1 = min(rows, r0 + step // d_qk)
        kv[r0:r1] = torch.randn(r1 - r0, d_qk, generator=g6, device=device).to(torch.bfloat16)
    return Workload(cfg_id=cfg_id, name=name or f"decode_B{batch}", mode="decode",
                    dims=dict(dims), softmax_scale=softmax_scale or 1.0 / math.sqrt(d_qk),
                    seqlens=lens, q_idx=q8, q_scale=qs, w=w.contiguous(), k_idx=k8,
                    k_scale=ks, q=q, kv=kv,
                    seq_lens=torch.tensor(lens, dtype=torch.int32, device=device),
                    block_table=block_table, max_seqlen=max_len)


def make_config(cfg_id: int, device="cpu", seed: Optional[int] = None) -> Workload:
    c = CONFIGS[cfg_id]
    dims = {k: c[k] for k in ("h_idx", "d_idx", "topk", "h", "d_qk", "d_v")}
    if c["mode"] == "prefill":
        return make_prefill(cfg_id, c["seqlens"], dims, c["needles"], device, seed=seed,
                            name=c["name"])
    return make_decode(cfg_id, c["batch"], c["ctx"], dims, c["boost"], c["paged"], device,
                       seed=seed, name=c["name"], scale_layout=c.get("scale_layout", "separate"))


def sample_rows(w: Workload, per_seq: int, first: int = 0, seed: Optional[int] = None
                ) -> List[int]:
    """Seeded sample of packed query rows: ``per_seq`` rows drawn per sequence plus every row
    with position < ``first``.  Returned sorted."""
    import numpy as np
    rng = np.random.default_rng((1000 + w.cfg_id if seed is None else seed) + 1)
    rows = set()
    off = 0
    for L in w.seqlens:
        n = min(per_seq, L)
        rows.update((off + rng.choice(L, size=n, replace=False)).tolist())
        rows.update(range(off, off + min(first, L)))
        off += L
    return sorted(int(r) for r in rows)
