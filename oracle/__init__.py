"""CPU oracle for the DSA hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The product path (``sparse_attention_long_04_b200``) never does, and
this package never imports the product path: the two share no code.  Inputs come from the
seeded generators in ``dsa_workloads``, which hold none of the method's arithmetic.

Stages (the pages' order: "FP8 index -> top-k selection -> sparse core attention",
"DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek Sparse Attention (DSA)", pipeline
summary):

  indexer_rows      S[t,s] = s_k[s] sum_j w[t,j] s_q[t,j] ReLU(q[t,j].k[s]),  s <= pos(t)
  topk_rows         k largest S per row, ties -> smaller index, all keys if fewer than k
  sparse_mla_rows   MQA-mode attention over the selected latent rows, fp64, with LSE
  quantize_e4m3     per-row e4m3 quantisation (scale = amax / 448), the decode cache append's
  cache_append      arithmetic; cache_append writes a decode step's new token into the caches
  kl_target_rows    the indexer's training target: the main attention's head-summed distribution
                    on the selected keys ("Training signal")
  indexer_kl_rows   KL(target || softmax of the indexer scores) and its gradients for w, q, k

The C library ``dsa_oracle.c`` does the arithmetic (OpenMP over rows); this module only
resolves which physical cache row holds logical key s of a sequence and moves bytes.

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against things other
than itself (the OCP FP8 spec values and torch's e4m3 cast, numpy matmul on the one-head
special case, hand-worked fixtures in ``tests/golden/``, brute-force sorting, torch's fp64
scaled-dot-product attention on the k >= context special case, and closed forms).
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Sequence

import numpy as np

from . import build as _build

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        f64p = ctypes.POINTER(ctypes.c_double)
        L.dsa_oracle_e4m3_to_f64.restype = ctypes.c_double
        L.dsa_oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.dsa_oracle_bf16_to_f64.restype = ctypes.c_double
        L.dsa_oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.dsa_oracle_indexer_seq.restype = None
        L.dsa_oracle_indexer_seq.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int64, f64p, ctypes.c_int]
        L.dsa_oracle_topk.restype = None
        L.dsa_oracle_topk.argtypes = [ctypes.c_int, ctypes.c_int, f64p, ctypes.c_int64,
                                      ctypes.c_void_p, ctypes.c_void_p]
        L.dsa_oracle_sparse_mla.restype = None
        L.dsa_oracle_sparse_mla.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, f64p, f64p]
        L.dsa_oracle_quantize_e4m3.restype = None
        L.dsa_oracle_quantize_e4m3.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_void_p]
        L.dsa_oracle_attn_target.restype = None
        L.dsa_oracle_attn_target.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, f64p]
        L.dsa_oracle_indexer_kl.restype = None
        L.dsa_oracle_indexer_kl.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, f64p, f64p, f64p,
            ctypes.c_void_p, f64p, f64p, f64p, f64p, f64p, f64p]
        L.dsa_oracle_num_threads.restype = ctypes.c_int
        _LIB = L
    return _LIB


def num_threads() -> int:
    return int(lib().dsa_oracle_num_threads())


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _np(t, dtype=None) -> np.ndarray:
    """torch tensor / numpy array -> contiguous numpy (bf16 tensors as uint16 bit patterns)."""
    if t is None:
        return None
    if hasattr(t, "detach"):
        import torch
        t = t.detach().cpu()
        if t.dtype == torch.bfloat16:
            t = t.view(torch.int16)
            return np.ascontiguousarray(t.numpy().view(np.uint16))
        if t.dtype == torch.float8_e4m3fn:
            t = t.view(torch.uint8)
        t = t.numpy()
    a = np.ascontiguousarray(t)
    return a.astype(dtype) if dtype is not None and a.dtype != dtype else a


def _take(t, rows, dtype=None) -> np.ndarray:
    """Rows ``rows`` of a torch tensor (gathered where it lives, then copied to the host) or of
    a numpy array; bf16 comes back as uint16 bit patterns."""
    rows = np.asarray(rows, dtype=np.int64)
    if hasattr(t, "detach"):
        import torch
        idx = torch.as_tensor(rows, device=t.device)
        return _np(t.index_select(0, idx), dtype)
    return _np(np.asarray(t)[rows], dtype)


def e4m3_to_f64(byte: int) -> float:
    return float(lib().dsa_oracle_e4m3_to_f64(int(byte)))


def bf16_to_f64(bits: int) -> float:
    return float(lib().dsa_oracle_bf16_to_f64(int(bits)))


# ---- sequence geometry ------------------------------------------------------------------

class Geometry:
    """Where each query row and each logical key lives.

    prefill: packed rows; row r of sequence b (cu[b] <= r < cu[b+1]) has position r - cu[b];
             logical key s of sequence b is physical row cu[b] + s.
    decode : row b is the new token of sequence b at position seq_lens[b] - 1; logical key s
             is physical row block_table[b, s // bs] * bs + s % bs when a block table is
             given, else b * max_seqlen + s.
    """

    def __init__(self, mode: str, seqlens: Sequence[int], block_table=None,
                 max_seqlen: int = 0, block_size: int = 64):
        self.mode = mode
        self.seqlens = [int(x) for x in seqlens]
        self.block_table = _np(block_table)
        self.max_seqlen = int(max_seqlen) or max(self.seqlens)
        self.block_size = block_size
        self.cu = np.concatenate([[0], np.cumsum(self.seqlens)]).astype(np.int64)

    @classmethod
    def of(cls, wl) -> "Geometry":
        return cls(wl.mode, wl.seqlens, wl.block_table, wl.max_seqlen)

    def row_seq_pos(self, row: int):
        if self.mode == "decode":
            return row, self.seqlens[row] - 1
        b = int(np.searchsorted(self.cu, row, side="right") - 1)
        return b, int(row - self.cu[b])

    def phys(self, b: int, s: np.ndarray) -> np.ndarray:
        s = np.asarray(s, dtype=np.int64)
        if self.mode == "prefill":
            return self.cu[b] + s
        if self.block_table is not None:
            bs = self.block_size
            return self.block_table[b, s // bs].astype(np.int64) * bs + s % bs
        return b * self.max_seqlen + s


def key_rows(wl, phys) -> tuple:
    """e4m3 codes [n, d_idx] and fp32 scales [n] of the indexer keys at physical rows
    ``phys``, from separate arrays or, when ``wl.k_scale`` is None, from 64-row blocks that
    hold their key rows followed by their scales."""
    phys = np.asarray(phys, dtype=np.int64)
    if wl.k_scale is not None:
        return _take(wl.k_idx, phys, np.uint8), _take(wl.k_scale, phys, np.float32)
    d = wl.dims["d_idx"]
    blk, j = phys // 64, phys % 64
    ub, inv = np.unique(blk, return_inverse=True)
    blocks = _take(wl.k_idx, ub, np.uint8)[inv]                  # [n, 64 * (d + 4)]
    n = len(phys)
    rows = np.arange(n)[:, None]
    codes = blocks[rows, j[:, None] * d + np.arange(d)[None, :]]
    sbytes = np.ascontiguousarray(blocks[rows, 64 * d + j[:, None] * 4 + np.arange(4)[None, :]])
    return np.ascontiguousarray(codes), sbytes.view(np.float32).reshape(n)


# ---- stages --------------------------------------------------------------------------------

def indexer_rows(wl, rows: Sequence[int], fp32: bool = False) -> Dict[int, np.ndarray]:
    """Scores of each packed query row against keys 0..pos(row) of its sequence.
    Returns {row: float64 array of length pos+1}."""
    geo = Geometry.of(wl)
    d = wl.dims
    h_idx, d_idx = d["h_idx"], d["d_idx"]
    by_seq: Dict[int, List[int]] = {}
    for r in rows:
        b, _ = geo.row_seq_pos(r)
        by_seq.setdefault(b, []).append(int(r))
    out: Dict[int, np.ndarray] = {}
    for b, rs in by_seq.items():
        pos = np.array([geo.row_seq_pos(r)[1] for r in rs], dtype=np.int32)
        n_keys = int(pos.max()) + 1
        phys = geo.phys(b, np.arange(n_keys))
        kseq, kss = key_rows(wl, phys)
        qq = _take(wl.q_idx, rs, np.uint8)
        qsc = _take(wl.q_scale, rs, np.float32)
        ww = _take(wl.w, rs, np.float32)
        res = np.full((len(rs), n_keys), np.nan, dtype=np.float64)
        lib().dsa_oracle_indexer_seq(len(rs), h_idx, d_idx, _ptr(qq), _ptr(qsc), _ptr(ww),
                                     _ptr(pos), n_keys, _ptr(kseq), _ptr(kss), n_keys,
                                     _f64p(res), 1 if fp32 else 0)
        for i, r in enumerate(rs):
            out[r] = res[i, : pos[i] + 1].copy()
    return out


def topk_rows(scores: Sequence[np.ndarray], topk: int) -> np.ndarray:
    """Selection per row under (score descending, index ascending); -1 padded.
    Returns int32 [n_rows, topk] in selection order."""
    n = len(scores)
    ld = max(1, max((len(s) for s in scores), default=1))
    mat = np.zeros((n, ld), dtype=np.float64)
    nv = np.zeros(n, dtype=np.int32)
    for i, s in enumerate(scores):
        mat[i, : len(s)] = s
        nv[i] = len(s)
    idx = np.empty((n, topk), dtype=np.int32)
    lib().dsa_oracle_topk(n, topk, _f64p(mat), ld, _ptr(nv), _ptr(idx))
    return idx


def sparse_mla_rows(wl, rows: Sequence[int], idx: np.ndarray):
    """Attention of each packed query row over its selected logical keys ``idx`` (int32
    [n_rows, k], -1 = unused).  Returns (O float64 [n, h, d_v], LSE float64 [n, h])."""
    geo = Geometry.of(wl)
    d = wl.dims
    h, d_qk, d_v = d["h"], d["d_qk"], d["d_v"]
    idx = np.asarray(idx)
    k = idx.shape[1]
    phys = np.full(idx.shape, -1, dtype=np.int64)
    for i, r in enumerate(rows):
        b, _ = geo.row_seq_pos(r)
        sel = idx[i] >= 0
        phys[i, sel] = geo.phys(b, idx[i, sel])
    qq = _take(wl.q, list(rows))
    # only the selected latent rows travel: remap physical rows to a compact host array
    used = np.unique(phys[phys >= 0])
    kv = _take(wl.kv, used) if len(used) else np.zeros((1, d_qk), np.uint16)
    compact = np.full(phys.shape, -1, dtype=np.int64)
    compact[phys >= 0] = np.searchsorted(used, phys[phys >= 0])
    phys = compact
    out = np.empty((len(rows), h, d_v), dtype=np.float64)
    lse = np.empty((len(rows), h), dtype=np.float64)
    lib().dsa_oracle_sparse_mla(len(rows), h, d_qk, d_v, float(wl.softmax_scale), _ptr(qq),
                                _ptr(kv), _ptr(phys), k, _f64p(out), _f64p(lse))
    return out, lse


def forward_rows(wl, rows: Sequence[int]):
    """All three stages for the given rows: (scores dict, idx, O, LSE)."""
    sc = indexer_rows(wl, rows)
    idx = topk_rows([sc[r] for r in rows], wl.dims["topk"])
    o, lse = sparse_mla_rows(wl, rows, idx)
    return sc, idx, o, lse


# ---- indexer training signal -----------------------------------------------------------------

def _selected_phys(geo, rows, idx):
    """Physical cache rows of the selected logical keys (-1 where idx < 0)."""
    phys = np.full(idx.shape, -1, dtype=np.int64)
    for i, r in enumerate(rows):
        b, _ = geo.row_seq_pos(r)
        sel = idx[i] >= 0
        phys[i, sel] = geo.phys(b, idx[i, sel])
    return phys


def kl_target_rows(wl, rows: Sequence[int], idx: np.ndarray) -> np.ndarray:
    """The indexer's training target on the selected keys: the main attention's distribution
    summed over heads and normalised (mean over heads of each head's softmax), float64
    [n_rows, k]; 0 where idx < 0."""
    geo = Geometry.of(wl)
    d = wl.dims
    idx = np.asarray(idx)
    k = idx.shape[1]
    phys = _selected_phys(geo, rows, idx)
    qq = _take(wl.q, list(rows))
    used = np.unique(phys[phys >= 0])
    kv = _take(wl.kv, used) if len(used) else np.zeros((1, d["d_qk"]), np.uint16)
    compact = np.full(phys.shape, -1, dtype=np.int64)
    compact[phys >= 0] = np.searchsorted(used, phys[phys >= 0])
    out = np.empty((len(rows), k), dtype=np.float64)
    lib().dsa_oracle_attn_target(len(rows), d["h"], d["d_qk"], float(wl.softmax_scale),
                                 _ptr(qq), _ptr(kv), _ptr(compact), k, _f64p(out))
    return out


def _e4m3_table() -> np.ndarray:
    return np.array([e4m3_to_f64(b) for b in range(256)], dtype=np.float64)


def indexer_kl_rows(wl, rows: Sequence[int], idx: np.ndarray, target: np.ndarray) -> dict:
    """KL(target || softmax of the indexer scores) on the selected keys of each row, and its
    gradients with respect to the indexer weights w, the real-valued indexer queries
    (s_q * q-hat) and the real-valued indexer keys (s_k * k-hat).  Returns float64 arrays:
    loss [n], scores [n, k], dw [n, h_idx], dq [n, h_idx, d_idx], and dk [u, d_idx] summed
    over the given rows for the physical key rows dk_rows [u]."""
    geo = Geometry.of(wl)
    d = wl.dims
    h_idx, d_idx = d["h_idx"], d["d_idx"]
    idx = np.asarray(idx)
    n, k = idx.shape
    tab = _e4m3_table()
    qc = _take(wl.q_idx, list(rows), np.uint8).reshape(n, h_idx, d_idx)
    qs = _take(wl.q_scale, list(rows), np.float32).reshape(n, h_idx).astype(np.float64)
    q = np.ascontiguousarray(tab[qc] * qs[:, :, None])
    w = np.ascontiguousarray(_take(wl.w, list(rows), np.float32).reshape(n, h_idx), np.float64)
    phys = _selected_phys(geo, rows, idx)
    valid = (phys >= 0).astype(np.int32)
    keys = np.zeros((n, k, d_idx), dtype=np.float64)
    if valid.any():
        codes, scales = key_rows(wl, phys[phys >= 0])
        keys[phys >= 0] = tab[codes] * scales.astype(np.float64)[:, None]
    res = indexer_kl_real(q, w, keys, valid, target)
    dk_rows, inv = np.unique(phys[phys >= 0], return_inverse=True)
    dk = np.zeros((len(dk_rows), d_idx))
    np.add.at(dk, inv, res.pop("dk")[phys >= 0])
    res.update(dk_rows=dk_rows, dk=dk)
    return res


def indexer_kl_real(q, w, keys, valid, target) -> dict:
    """The same loss and gradients on real-valued inputs given directly (float64 q [n, h, d],
    w [n, h], keys [n, k, d], valid [n, k], target [n, k]); dk is per selected entry,
    [n, k, d]."""
    q = np.ascontiguousarray(q, np.float64)
    w = np.ascontiguousarray(w, np.float64)
    keys = np.ascontiguousarray(keys, np.float64)
    valid = np.ascontiguousarray(valid, np.int32)
    tgt = np.ascontiguousarray(target, np.float64)
    n, h_idx, d_idx = q.shape
    k = keys.shape[1]
    loss = np.empty(n)
    scores = np.empty((n, k))
    dw = np.empty((n, h_idx))
    dq = np.empty((n, h_idx, d_idx))
    dkeys = np.empty((n, k, d_idx))
    lib().dsa_oracle_indexer_kl(n, h_idx, d_idx, k, _f64p(q), _f64p(w), _f64p(keys),
                                _ptr(valid), _f64p(tgt), _f64p(loss), _f64p(scores),
                                _f64p(dw), _f64p(dq), _f64p(dkeys))
    return dict(loss=loss, scores=scores, dw=dw, dq=dq, dk=dkeys)


# ---- decode cache append ---------------------------------------------------------------------

def quantize_e4m3(x) -> tuple:
    """Per-row e4m3 codes and fp32 scales of fp32 rows ``x`` [n, d] (the "FP8 index" input
    format: one scale per token).  Returns (uint8 [n, d], float32 [n])."""
    x = np.ascontiguousarray(_np(x), dtype=np.float32)
    n, d = x.shape
    codes = np.empty((n, d), dtype=np.uint8)
    scales = np.empty(n, dtype=np.float32)
    lib().dsa_oracle_quantize_e4m3(n, d, _ptr(x), _ptr(codes), _ptr(scales))
    return codes, scales


def cache_append(k_cache, k_scale, kv_cache, seq_lens, block_table, max_seqlen: int,
                 k_new, kv_new, block_size: int = 64):
    """One decode step's append: for each sequence b the new token sits at position
    p = seq_lens[b] - 1; its indexer key k_new[b] (fp32) is quantised per token and written
    with its scale, and its latent row kv_new[b] (bf16 bits) is copied, at the physical row
    block_table[b, p // bs] * bs + p % bs (b * max_seqlen + p without a table).  Entries
    whose position or block is outside the caches are skipped.  With ``k_scale`` None the key
    cache is made of 64-row blocks holding their key rows then their fp32 scales.  Returns
    copies of the three caches (the scales None in that layout) and a bool [B] of the skipped
    entries."""
    kc, kv = _np(k_cache).copy(), _np(kv_cache).copy()
    ks = _np(k_scale).copy() if k_scale is not None else None    # None: scales in the blocks
    lens = _np(seq_lens).astype(np.int64)
    bt = _np(block_table)
    codes, scales = quantize_e4m3(k_new)
    kvn = _np(kv_new)
    rows = kv.shape[0]
    bad = np.zeros(len(lens), dtype=bool)
    for b, n in enumerate(lens):
        p = int(n) - 1
        if p < 0 or p >= max_seqlen:
            bad[b] = True
            continue
        if bt is not None:
            blk = int(bt[b, p // block_size])
            phys = blk * block_size + p % block_size
            if blk < 0 or (blk + 1) * block_size > rows:
                bad[b] = True
                continue
        else:
            phys = b * max_seqlen + p
            if phys >= rows:
                bad[b] = True
                continue
        if ks is not None:
            kc[phys] = codes[b]
            ks[phys] = scales[b]
        else:                                   # block phys // 64: 64 key rows, then scales
            d = codes.shape[1]
            blk, j = phys // 64, phys % 64
            kc[blk, j * d:(j + 1) * d] = codes[b]
            kc[blk, 64 * d + 4 * j:64 * d + 4 * j + 4] = np.frombuffer(
                scales[b:b + 1].tobytes(), dtype=np.uint8)
        kv[phys] = kvn[b]
    return kc, ks, kv, bad
