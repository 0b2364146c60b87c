"""NumPy twin of the C oracle, for tiny inputs -- TEST INFRASTRUCTURE ONLY.

Vectorised fp64 restatements of the same definitions (indexer, top-k, MQA-mode sparse
attention, and the indexer's training target and KL gradients; "DeepSeek V3.2-Exp Cuts
Long-Context Costs with DeepSeek Sparse Attention (DSA)", pipeline summary, "Instantiation" and
"Training signal").  Written independently of ``dsa_oracle.c`` so that the
two cross-check each other; neither is the CUDA path.
"""
from __future__ import annotations

import numpy as np


def e4m3_table() -> np.ndarray:
    """All 256 e4m3 codes decoded from the field definitions (sign, 4-bit exponent with bias
    7, 3-bit mantissa, subnormals at exponent 0, S.1111.111 = NaN)."""
    b = np.arange(256)
    sign = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    v = sign * np.where(e == 0, sub, normal)
    v[(e == 15) & ((b & 7) == 7)] = np.nan
    return v


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def indexer(q8, q_scale, w, k8, k_scale) -> np.ndarray:
    """All-pairs scores, no causal mask: q8 [T, H_I, D_I] codes, k8 [N, D_I] codes.
    Returns [T, N] = s_k * sum_j (w * s_q)[t, j] * max(q[t, j] . k, 0)."""
    tab = e4m3_table()
    q = tab[np.asarray(q8, dtype=np.int64)]
    k = tab[np.asarray(k8, dtype=np.int64)]
    dots = np.einsum("tjd,nd->tjn", q, k)
    coef = np.asarray(w, np.float64) * np.asarray(q_scale, np.float64)
    return np.einsum("tj,tjn->tn", coef, np.maximum(dots, 0.0)) * np.asarray(k_scale,
                                                                             np.float64)[None]


def topk(scores: np.ndarray, k: int) -> np.ndarray:
    """Selected indices of one row in selection order (lexsort on (index, -score))."""
    s = np.asarray(scores, dtype=np.float64)
    order = np.lexsort((np.arange(len(s)), -s))
    sel = order[:k]
    return np.concatenate([sel, -np.ones(max(0, k - len(sel)), dtype=np.int64)])


def sparse_attention(q_bits, kv_bits, sel_rows, scale: float, d_v: int):
    """q_bits [H, D_qk] bf16 codes of one query row; kv_bits [R, D_qk]; sel_rows physical
    rows (-1 ignored).  Returns (O [H, d_v], LSE [H])."""
    q = bf16_to_f64(q_bits)
    sel = np.asarray([s for s in sel_rows if s >= 0], dtype=np.int64)
    kv = bf16_to_f64(kv_bits[sel])
    logits = scale * (q @ kv.T)                     # [H, n]
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    den = p.sum(axis=1, keepdims=True)
    return (p @ kv[:, :d_v]) / den, (m + np.log(den))[:, 0]


def kl_target(q_bits, kv_bits, sel_rows, scale: float) -> np.ndarray:
    """The indexer's training target on one row's selection: the mean over heads of each
    head's softmax over the selected latent rows ("Training signal").  q_bits [H, D_qk],
    kv_bits [R, D_qk] bf16 codes; sel_rows physical rows (-1: unused, target 0)."""
    sel_rows = np.asarray(sel_rows, dtype=np.int64)
    out = np.zeros(len(sel_rows))
    used = sel_rows >= 0
    if not used.any():
        return out
    q = bf16_to_f64(q_bits)
    kv = bf16_to_f64(kv_bits[sel_rows[used]])
    logits = scale * (q @ kv.T)                      # [H, n]
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    out[used] = p.mean(axis=0)
    return out


def indexer_kl(q, w, keys, valid, target):
    """KL(target || softmax of the indexer scores) on one row's selection and its gradients,
    written with whole-array operations: q [H_I, D_I], w [H_I], keys [k, D_I] real-valued,
    valid [k] bool, target [k].  Returns (loss, dw [H_I], dq [H_I, D_I], dk [k, D_I])."""
    q, w, keys = (np.asarray(a, np.float64) for a in (q, w, keys))
    valid = np.asarray(valid, bool)
    p = np.where(valid, np.asarray(target, np.float64), 0.0)
    dots = q @ keys.T                                # [H_I, k]
    relu = np.maximum(dots, 0.0)
    s = np.where(valid, w @ relu, -np.inf)
    log_pi = s - (s.max() + np.log(np.exp(s - s.max()).sum())) if valid.any() else s
    pi = np.where(valid, np.exp(log_pi), 0.0)
    pos = p > 0
    loss = float((p[pos] * (np.log(p[pos]) - log_pi[pos])).sum())
    g = np.where(valid, pi * p.sum() - p, 0.0)
    gate = (dots > 0).astype(np.float64)             # d ReLU / d x, 0 at x = 0
    dw = relu @ g
    dq = (w[:, None] * (gate * g[None, :])) @ keys
    dk = (g[:, None] * (gate.T * w[None, :])) @ q
    return loss, dw, dq, dk
