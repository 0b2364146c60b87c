"""Pins for the CPU oracle: each check ties it to something other than itself.

Runs without a GPU.  Sources of truth used here: the OCP FP8 E4M3 field definition and
torch's float8_e4m3fn cast; numpy matmul (the one-head, unit-weight special case of the
indexer); hand-worked fixtures under tests/golden/; brute-force sorting; torch's fp64
scaled_dot_product_attention and logsumexp (the k >= context special case); closed forms.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import reference_np
from dsa_workloads import make_prefill, make_decode, quantize_e4m3_rows

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- input decoding

def test_e4m3_spec_values():
    # OCP FP8 E4M3: max finite 448 (0x7E), min subnormal 2^-9 (0x01), min normal 2^-6 (0x08),
    # 1.0 = 0x38, NaN = 0x7F / 0xFF, negative zero 0x80
    assert oracle.e4m3_to_f64(0x7E) == 448.0
    assert oracle.e4m3_to_f64(0xFE) == -448.0
    assert oracle.e4m3_to_f64(0x01) == 2.0 ** -9
    assert oracle.e4m3_to_f64(0x07) == 7 * 2.0 ** -9
    assert oracle.e4m3_to_f64(0x08) == 2.0 ** -6
    assert oracle.e4m3_to_f64(0x38) == 1.0
    assert oracle.e4m3_to_f64(0x39) == 1.125
    assert math.isnan(oracle.e4m3_to_f64(0x7F)) and math.isnan(oracle.e4m3_to_f64(0xFF))
    assert math.copysign(1.0, oracle.e4m3_to_f64(0x80)) == -1.0


def test_e4m3_all_codes_match_torch_cast():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle.e4m3_to_f64(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine))
    assert np.array_equal(ref[~nan], mine[~nan])
    tw = reference_np.e4m3_table()
    assert np.array_equal(np.isnan(tw), nan) and np.array_equal(tw[~nan], ref[~nan])


def test_bf16_decode_matches_torch():
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(4096, generator=g) * 1e3).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    mine = np.array([oracle.bf16_to_f64(b) for b in bits[:512]])
    assert np.array_equal(mine, x[:512].to(torch.float64).numpy())
    assert np.array_equal(reference_np.bf16_to_f64(bits), x.to(torch.float64).numpy())


# ---------------------------------------------------------------- indexer

class _W:
    """Minimal workload stand-in for the oracle's duck-typed inputs."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def _one_seq(q8, qs, w, k8, ks, h_idx, d_idx, d=None):
    T = q8.shape[0]
    return _W(mode="prefill", seqlens=[T], block_table=None, max_seqlen=T,
              dims=dict(h_idx=h_idx, d_idx=d_idx, **(d or {})), q_idx=q8, q_scale=qs, w=w,
              k_idx=k8, k_scale=ks)


def test_indexer_hand_fixture():
    g = _load("indexer_hand.json")
    q8 = np.array([g["q_codes"]], dtype=np.uint8)              # one query row
    k8 = np.array(g["k_codes"], dtype=np.uint8)
    # the codes decode to the stated values (pins the fixture itself)
    dec = torch.from_numpy(k8).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(dec, np.array(g["k_values"], dtype=np.float64))
    # query row sits at position pos = 2 of a 3-token sequence: pad with two dummy rows
    q8 = np.concatenate([np.zeros((2, 2, 4), np.uint8), q8])
    qs = np.array([[1, 1], [1, 1], g["q_scale"]], np.float32)
    w = np.array([[0, 0], [0, 0], g["w"]], np.float32)
    wl = _one_seq(q8, qs, w, k8, np.array(g["k_scale"], np.float32), 2, 4)
    for fp32 in (False, True):
        got = oracle.indexer_rows(wl, [2], fp32=fp32)[2]
        assert np.array_equal(got, np.array(g["expected"]))
    # causality: the row at position 1 sees keys 0..1 only
    assert len(oracle.indexer_rows(wl, [1])[1]) == 2


def test_indexer_one_head_is_relu_matmul():
    rng = np.random.default_rng(0)
    T, D = 37, 32
    q = torch.from_numpy(rng.standard_normal((T, 1, D)) * 4).float()
    k = torch.from_numpy(rng.standard_normal((T, D)) * 4).float()
    q8 = q.to(torch.float8_e4m3fn)
    k8 = k.to(torch.float8_e4m3fn)
    ones_q = np.ones((T, 1), np.float32)
    wl = _one_seq(q8.view(torch.uint8).numpy(), ones_q, ones_q, k8.view(torch.uint8).numpy(),
                  np.ones(T, np.float32), 1, D)
    ref = np.maximum(q8.double().numpy()[:, 0, :] @ k8.double().numpy().T, 0.0)  # numpy matmul
    got = oracle.indexer_rows(wl, list(range(T)))
    for t in range(T):
        assert np.array_equal(got[t], ref[t, : t + 1])


def test_indexer_scale_homogeneity_and_head_additivity():
    rng = np.random.default_rng(1)
    T, H, D = 20, 3, 32
    q8 = rng.integers(0, 256, (T, H, D), dtype=np.uint8)
    q8[(q8 & 0x7F) == 0x7F] = 0x38                   # no NaN codes
    k8 = rng.integers(0, 256, (T, D), dtype=np.uint8)
    k8[(k8 & 0x7F) == 0x7F] = 0x38
    qs = rng.uniform(0.5, 2, (T, H)).astype(np.float32)
    w = rng.uniform(0, 1, (T, H)).astype(np.float32)
    ks = rng.uniform(0.5, 2, T).astype(np.float32)
    base = oracle.indexer_rows(_one_seq(q8, qs, w, k8, ks, H, D), range(T))
    scaled = oracle.indexer_rows(_one_seq(q8, qs * 2, w * 4, k8, ks * 0.5, H, D), range(T))
    for t in range(T):
        assert np.array_equal(scaled[t], base[t] * 4.0)       # powers of two: exact
    # additivity over heads: S(all heads) = sum_j S(head j alone)
    tot = np.zeros(T)
    parts = [oracle.indexer_rows(_one_seq(np.ascontiguousarray(q8[:, j:j + 1]),
                                          np.ascontiguousarray(qs[:, j:j + 1]),
                                          np.ascontiguousarray(w[:, j:j + 1]), k8, ks, 1, D),
                                 [T - 1])[T - 1] for j in range(H)]
    np.testing.assert_allclose(base[T - 1], sum(parts), rtol=1e-12, atol=0)
    # and each part really is one head: a head with weight 0 contributes nothing
    w0 = w.copy()
    w0[:, 1] = 0
    no1 = oracle.indexer_rows(_one_seq(q8, qs, w0, k8, ks, H, D), [T - 1])[T - 1]
    np.testing.assert_allclose(no1, parts[0] + parts[2], rtol=1e-12, atol=0)


def test_indexer_fp32_path_close_to_fp64_and_numpy_twin():
    wl = make_prefill(99, [300], dict(h_idx=4, d_idx=32, topk=64, h=4, d_qk=32, d_v=16),
                      needles=8, device="cpu", seed=5)
    rows = [0, 1, 127, 128, 299]
    a = oracle.indexer_rows(wl, rows)
    b = oracle.indexer_rows(wl, rows, fp32=True)
    tw = reference_np.indexer(wl.q_idx.numpy(), wl.q_scale.numpy(), wl.w.numpy(),
                              wl.k_idx.numpy(), wl.k_scale.numpy())
    for r in rows:
        np.testing.assert_allclose(b[r], a[r], rtol=1e-5, atol=1e-6 * a[r].max())
        np.testing.assert_allclose(a[r], tw[r, : r + 1], rtol=1e-12, atol=1e-12)


def test_paged_geometry_hand_and_equivalence():
    geo = oracle.Geometry("decode", [100], block_table=np.array([[3, 1]]), max_seqlen=100)
    assert geo.phys(0, np.array([5, 70])).tolist() == [3 * 64 + 5, 1 * 64 + 6]
    dims = dict(h_idx=4, d_idx=32, topk=64, h=4, d_qk=32, d_v=16)
    wp = make_decode(98, 3, [130, 64, 200], dims, boost=0.05, paged=True, device="cpu",
                     seed=11, total_blocks=20)
    # the same data laid out contiguously per sequence (gathered here with torch indexing)
    bt = wp.block_table.long()
    L = max(wp.seqlens)
    idx = torch.stack([bt[b, torch.arange(L) // 64] * 64 + torch.arange(L) % 64
                       for b in range(3)]).reshape(-1)
    wc = _W(**{**wp.__dict__, "block_table": None, "k_idx": wp.k_idx[idx],
               "k_scale": wp.k_scale[idx], "kv": wp.kv[idx]})
    a = oracle.indexer_rows(wp, [0, 1, 2])
    c = oracle.indexer_rows(wc, [0, 1, 2])
    for r in range(3):
        assert len(a[r]) == wp.seqlens[r]
        assert np.array_equal(a[r], c[r])


# ---------------------------------------------------------------- top-k

def test_topk_hand_fixture():
    for case in _load("topk_hand.json")["cases"]:
        got = oracle.topk_rows([np.array(case["scores"], float)], case["k"])[0]
        assert got.tolist() == case["expected"], case


@pytest.mark.parametrize("ties", [False, True])
def test_topk_brute_force(ties):
    rng = np.random.default_rng(7 + ties)
    rows = []
    for n in [1, 5, 63, 64, 65, 500, 3000]:
        s = rng.integers(0, 6, n).astype(float) if ties else rng.standard_normal(n)
        rows.append(s)
    k = 64
    got = oracle.topk_rows(rows, k)
    for s, g in zip(rows, got):
        brute = sorted(range(len(s)), key=lambda i: (-s[i], i))[:k]
        assert g.tolist() == brute + [-1] * (k - len(brute))
        assert g.tolist() == reference_np.topk(s, k).tolist()


def test_topk_permutation_invariance_tie_free():
    rng = np.random.default_rng(8)
    s = rng.standard_normal(5000)
    assert len(np.unique(s)) == len(s)
    perm = rng.permutation(len(s))
    a = set(oracle.topk_rows([s], 100)[0].tolist())
    b = oracle.topk_rows([s[perm]], 100)[0]
    assert set(perm[b].tolist()) == a


# ---------------------------------------------------------------- sparse attention

def _tiny_attn_workload(L=40, h=4, d_qk=24, d_v=16, seed=2):
    return make_prefill(97, [L], dict(h_idx=4, d_idx=32, topk=8, h=h, d_qk=d_qk, d_v=d_v),
                        needles=0, device="cpu", seed=seed, softmax_scale=0.3)


def test_attention_full_set_equals_torch_sdpa_causal_mqa():
    wl = _tiny_attn_workload()
    L, h, d_v = 40, 4, 16
    rows = list(range(L))
    idx = np.array([list(range(t + 1)) + [-1] * (L - t - 1) for t in rows], np.int32)
    o, lse = oracle.sparse_mla_rows(wl, rows, idx)
    q = wl.q.double().permute(1, 0, 2)                  # [h, L, d_qk]
    kv = wl.kv.double()
    k = kv.unsqueeze(0).expand(h, -1, -1)               # MQA: one KV row shared by all heads
    v = kv[:, :d_v].unsqueeze(0).expand(h, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=0.3)
    np.testing.assert_allclose(o, ref.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    logits = torch.matmul(q, k.transpose(1, 2)) * 0.3
    logits = logits.masked_fill(torch.triu(torch.ones(L, L, dtype=torch.bool), 1), -math.inf)
    ref_lse = torch.logsumexp(logits, dim=-1).permute(1, 0).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_attention_k1_and_identical_rows_closed_forms():
    wl = _tiny_attn_workload()
    qd = wl.q.double().numpy()
    kvd = wl.kv.double().numpy()
    # k = 1: output is that row's value part, LSE is its scaled logit
    o, lse = oracle.sparse_mla_rows(wl, [30], np.array([[17, -1, -1]], np.int32))
    assert np.array_equal(o[0], np.broadcast_to(kvd[17, :16], (4, 16)))
    np.testing.assert_allclose(lse[0], 0.3 * qd[30] @ kvd[17], rtol=1e-13)
    # n identical rows: output that row, LSE = ln n + logit
    o, lse = oracle.sparse_mla_rows(wl, [30], np.array([[9] * 5], np.int32))
    np.testing.assert_allclose(o[0], np.broadcast_to(kvd[9, :16], (4, 16)), rtol=1e-14)
    np.testing.assert_allclose(lse[0], math.log(5) + 0.3 * qd[30] @ kvd[9], rtol=1e-13)


def test_attention_uniform_logit_shift():
    """Adding the same amount to every logit of a row leaves O unchanged and moves LSE by that
    amount: every key row gets 1 in a non-value dim, and the query's entry there goes from 0.5
    to 2.5 (both exact in bf16), a shift of 0.3 * 2 = 0.6 of each scaled logit."""
    wl = _tiny_attn_workload()
    wl.kv[:, 23] = 1.0                                  # d_qk = 24, d_v = 16: not a value dim
    wl.q[:, :, 23] = 0.5
    rows = [5, 30, 39]
    sel = np.array([[0, 1, 2, 3, 4, 5, -1, -1],
                    [3, 11, 0, 25, 7, 30, 29, 2],
                    [39, 38, 1, 12, -1, 20, 22, 9]], np.int32)
    o1, l1 = oracle.sparse_mla_rows(wl, rows, sel)
    wl.q[:, :, 23] = 2.5
    o2, l2 = oracle.sparse_mla_rows(wl, rows, sel)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l2, l1 + 0.6, rtol=1e-12, atol=1e-12)


def test_attention_order_and_padding_invariance_and_numpy_twin():
    wl = _tiny_attn_workload()
    sel = np.array([[3, 11, 0, 25, 7, 30, -1, -1]], np.int32)
    o1, l1 = oracle.sparse_mla_rows(wl, [30], sel)
    o2, l2 = oracle.sparse_mla_rows(wl, [30], np.array([[-1, 30, 7, -1, 25, 0, 11, 3]],
                                                       np.int32))
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(l1, l2, rtol=1e-13)
    qb = wl.q.view(torch.int16).numpy().view(np.uint16)[30]
    kvb = wl.kv.view(torch.int16).numpy().view(np.uint16)
    o3, l3 = reference_np.sparse_attention(qb, kvb, sel[0], 0.3, 16)
    np.testing.assert_allclose(o1[0], o3, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l1[0], l3, rtol=1e-12)


def test_attention_dense_masked_softmax_equals_sparse():
    """Dense attention with a top-k mask (numpy, all keys, -inf outside the set) equals the
    sparse oracle over the set."""
    wl = _tiny_attn_workload()
    qd = wl.q.double().numpy()[33]
    kvd = wl.kv.double().numpy()
    sel = [2, 5, 8, 13, 21, 33]
    logits = 0.3 * qd @ kvd[:34].T
    mask = np.full(34, -np.inf)
    mask[sel] = 0
    z = logits + mask
    p = np.exp(z - z.max(axis=1, keepdims=True))
    ref = (p / p.sum(axis=1, keepdims=True)) @ kvd[:34, :16]
    o, _ = oracle.sparse_mla_rows(wl, [33], np.array([sel], np.int32))
    np.testing.assert_allclose(o[0], ref, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- whole pipeline

def test_pipeline_rows_before_k_equal_dense_causal():
    """Rows with fewer than k prior tokens keep all of them, so the sparse result is dense
    causal MQA attention (torch fp64 SDPA)."""
    dims = dict(h_idx=4, d_idx=32, topk=64, h=4, d_qk=32, d_v=16)
    wl = make_prefill(96, [100], dims, needles=8, device="cpu", seed=4)
    rows = [0, 1, 30, 63]
    _, idx, o, lse = oracle.forward_rows(wl, rows)
    for i, t in enumerate(rows):
        assert sorted(idx[i][idx[i] >= 0].tolist()) == list(range(t + 1))
    q = wl.q.double().permute(1, 0, 2)[:, :64]
    kv = wl.kv.double()[:64]
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, kv.unsqueeze(0).expand(4, -1, -1), kv[:, :16].unsqueeze(0).expand(4, -1, -1),
        is_causal=True, scale=wl.softmax_scale).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(o, ref[rows], rtol=1e-10, atol=1e-12)


def test_workload_quantiser_roundtrip_bound():
    """The generator's e4m3 bytes decode to within half an e4m3 ulp (2^-4 relative) of the
    drawn values: the inputs the oracle and the kernels share are what they claim."""
    g = torch.Generator().manual_seed(0)
    x = torch.randn(64, 8, 32, generator=g)
    q8, s = quantize_e4m3_rows(x, 2)
    dec = q8.view(torch.float8_e4m3fn).double() * s.double()[:, None, None]
    err = (dec - x.double()).abs()
    amax = x.abs().amax(dim=(1, 2)).double()
    assert bool((err <= torch.maximum(x.double().abs() * 2 ** -4,
                                      (amax / 448 * 2 ** -9)[:, None, None] * 1.0001)).all())


# ---------------------------------------------------------------- decode cache append (e4m3)

def test_quantize_matches_torch_cast_and_generator():
    """Per-token e4m3 quantisation against an independent implementation: the generator's
    torch path (amax / 448, torch's round-to-nearest-even float8_e4m3fn cast)."""
    from dsa_workloads import quantize_e4m3_rows
    g = torch.Generator().manual_seed(31)
    rows = [torch.randn(64, 128, generator=g),
            torch.randn(64, 128, generator=g) ** 3 * 50,          # heavy tails
            torch.randn(8, 128, generator=g) * 1e-6,              # subnormal codes after scaling
            torch.full((2, 128), 3.25)]                            # constant rows
    for x in rows:
        ref_c, ref_s = quantize_e4m3_rows(x, 1)
        c, s = oracle.quantize_e4m3(x.numpy())
        assert np.array_equal(c, ref_c.numpy())
        assert np.array_equal(s, ref_s.numpy())


def test_quantize_ties_round_to_even():
    """Every midpoint between consecutive positive e4m3 values (exact in fp32) rounds to the
    neighbour with the even mantissa, like torch's cast; a 448 entry pins the scale to 1."""
    vals = sorted({oracle.e4m3_to_f64(b) for b in range(0x7F) if b != 0x7F})
    mids = [(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])]
    x = np.array(mids + [448.0], dtype=np.float32)
    c, s = oracle.quantize_e4m3(x[None, :])
    assert s[0] == 1.0
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(c[0], ref)
    assert all(int(v) & 1 == 0 for v in c[0, :-1])    # ties land on even mantissas


def test_quantize_error_bound_and_zero_row():
    """|x - e4m3(x / s) * s| <= half the e4m3 spacing at that magnitude (times s); an all-zero
    row has scale 1 and zero codes; the largest magnitude maps to +-448."""
    g = np.random.default_rng(5)
    x = g.standard_normal((16, 128)).astype(np.float32)
    c, s = oracle.quantize_e4m3(x)
    for r in range(16):
        dq = np.array([oracle.e4m3_to_f64(b) for b in c[r]]) * s[r]
        y = np.abs(x[r] / s[r]).astype(np.float64)
        spacing = np.where(y < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(y, 1e-30))) - 3))
        assert np.all(np.abs(dq - x[r]) <= 0.5 * spacing * s[r] * (1 + 1e-6))
        assert abs(oracle.e4m3_to_f64(c[r][np.argmax(np.abs(x[r]))])) == 448.0
    c0, s0 = oracle.quantize_e4m3(np.zeros((1, 128), np.float32))
    assert s0[0] == 1.0 and not c0.any()


def test_cache_append_paged_equals_contiguous():
    """The append writes each sequence's new token at position seq_len - 1 through its block
    table, touches nothing else, and reads back the same through a paged or a contiguous
    layout; entries whose position or block is outside the caches are skipped."""
    from dsa_workloads import make_decode, TINY
    dims = dict(TINY, h_idx=64, d_idx=128)
    lens = [130, 64, 1, 200]
    wl = make_decode(21, 4, lens, dims, boost=0.0, paged=True, device="cpu", total_blocks=20)
    g = np.random.default_rng(9)
    k_new = g.standard_normal((4, 128)).astype(np.float32)
    kv_new = (g.standard_normal((4, dims["d_qk"])).astype(np.float32).view(np.uint32) >> 16
              ).astype(np.uint16)
    kc, ks, kv, bad = oracle.cache_append(wl.k_idx, wl.k_scale, wl.kv, wl.seq_lens,
                                          wl.block_table, wl.max_seqlen, k_new, kv_new)
    assert not bad.any()
    codes, scales = oracle.quantize_e4m3(k_new)
    geo = oracle.Geometry.of(wl)
    changed = set()
    for b, n in enumerate(lens):
        phys = int(geo.phys(b, np.array([n - 1]))[0])
        changed.add(phys)
        assert np.array_equal(kc[phys], codes[b]) and ks[phys] == scales[b]
        assert np.array_equal(kv[phys], kv_new[b])
    keep = np.array([r for r in range(kc.shape[0]) if r not in changed])
    assert np.array_equal(kc[keep], oracle._np(wl.k_idx)[keep])
    assert np.array_equal(kv[keep], oracle._np(wl.kv)[keep])
    # contiguous layout: the same logical appends
    R = 4 * wl.max_seqlen
    z8, zs, z16 = (np.zeros((R, 128), np.uint8), np.ones(R, np.float32),
                   np.zeros((R, dims["d_qk"]), np.uint16))
    kc2, ks2, kv2, bad2 = oracle.cache_append(z8, zs, z16, wl.seq_lens, None, wl.max_seqlen,
                                              k_new, kv_new)
    for b, n in enumerate(lens):
        pp = int(geo.phys(b, np.array([n - 1]))[0])
        pc = b * wl.max_seqlen + n - 1
        assert np.array_equal(kc2[pc], kc[pp]) and ks2[pc] == ks[pp]
        assert np.array_equal(kv2[pc], kv[pp])
    # out-of-range entries are skipped
    bt = oracle._np(wl.block_table).copy()
    bt[0, 2] = -1
    lens_bad = np.array([130, 64, 0, 10_000], dtype=np.int32)
    _, _, _, bad3 = oracle.cache_append(wl.k_idx, wl.k_scale, wl.kv, lens_bad, bt,
                                        wl.max_seqlen, k_new, kv_new)
    assert list(bad3) == [True, False, True, True]


def test_interleaved_key_blocks_hold_the_same_keys():
    """A paged indexer cache whose 64-row blocks carry their own scales holds exactly the keys
    and scales of the separate layout (same seed), and an append lands on the same bytes."""
    from dsa_workloads import make_decode, FULL
    a = make_decode(62, 3, [700, 64, 200], FULL, boost=0.01, paged=True, device="cpu")
    b = make_decode(62, 3, [700, 64, 200], FULL, boost=0.01, paged=True, device="cpu",
                    scale_layout="interleaved")
    assert b.k_scale is None and b.k_idx.shape == (a.kv.shape[0] // 64, 64 * (128 + 4))
    phys = np.arange(a.kv.shape[0])
    ca, sa = oracle.key_rows(a, phys)
    cb, sb = oracle.key_rows(b, phys)
    assert np.array_equal(ca, cb) and np.array_equal(sa, sb)
    g = np.random.default_rng(4)
    k_new = g.standard_normal((3, 128)).astype(np.float32)
    kv_new = np.zeros((3, 576), np.uint16)
    ra = oracle.cache_append(a.k_idx, a.k_scale, a.kv, a.seq_lens, a.block_table,
                             a.max_seqlen, k_new, kv_new)
    rb = oracle.cache_append(b.k_idx, None, b.kv, b.seq_lens, b.block_table,
                             b.max_seqlen, k_new, kv_new)
    assert rb[1] is None
    a2 = type(a)(**{**a.__dict__, "k_idx": torch.from_numpy(ra[0]),
                    "k_scale": torch.from_numpy(ra[1])})
    b2 = type(b)(**{**b.__dict__, "k_idx": torch.from_numpy(rb[0])})
    c2a, s2a = oracle.key_rows(a2, phys)
    c2b, s2b = oracle.key_rows(b2, phys)
    assert np.array_equal(c2a, c2b) and np.array_equal(s2a, s2b)


# ---------------------------------------------------------------- indexer training signal

def test_kl_target_is_the_head_mean_of_the_attention_weights():
    """With no more selected keys than value dims, the head-mean of the attention outputs
    (pinned against torch's SDPA above) determines the head-mean of the attention weights:
    mean_h O[h] = sum_e t_e v_e.  The target must be that solution, sum to 1, and be 0 on
    unused slots."""
    wl = _tiny_attn_workload()
    kvd = wl.kv.double().numpy()
    rows = [30, 33, 39]
    idx = np.array([[3, 11, 0, -1, 25, 7, 30, -1],
                    [33, -1, 1, 2, 5, 8, 13, 21],
                    [39, 38, 37, 4, -1, -1, -1, -1]], np.int32)
    t = oracle.kl_target_rows(wl, rows, idx)
    o, _ = oracle.sparse_mla_rows(wl, rows, idx)
    for i in range(len(rows)):
        sel = idx[i] >= 0
        assert (t[i, ~sel] == 0).all()
        assert t[i].sum() == pytest.approx(1.0, abs=1e-13)
        v = kvd[idx[i, sel], :16]                        # [n_sel, d_v], independent rows
        sol, *_ = np.linalg.lstsq(v.T, o[i].mean(axis=0), rcond=None)
        np.testing.assert_allclose(t[i, sel], sol, rtol=1e-9, atol=1e-12)


def test_kl_target_closed_forms():
    wl = _tiny_attn_workload()
    t = oracle.kl_target_rows(wl, [30, 30], np.array([[-1, 17, -1], [9, 9, 9]], np.int32))
    assert list(t[0]) == [0.0, 1.0, 0.0]                # one key: all the mass
    np.testing.assert_allclose(t[1], [1 / 3] * 3, rtol=1e-14)   # identical keys: uniform
    assert not oracle.kl_target_rows(wl, [5], np.full((1, 4), -1, np.int32)).any()


def _kl_workload():
    dims = dict(h_idx=4, d_idx=32, topk=16, h=4, d_qk=24, d_v=16)
    return make_prefill(95, [60], dims, needles=4, device="cpu", seed=5, softmax_scale=0.3)


def test_indexer_kl_loss_is_scipy_kl_on_the_indexer_scores():
    """The loss is scipy's relative entropy of the target against the softmax of the indexer
    scores (those of the pinned indexer oracle) on each row's selected keys."""
    from scipy.special import softmax
    from scipy.stats import entropy
    wl = _kl_workload()
    rows = [3, 17, 40, 59]
    sc, idx, _, _ = oracle.forward_rows(wl, rows)
    target = oracle.kl_target_rows(wl, rows, idx)
    res = oracle.indexer_kl_rows(wl, rows, idx, target)
    for i, r in enumerate(rows):
        sel = idx[i] >= 0
        assert (res["scores"][i, ~sel] == -np.inf).all()
        np.testing.assert_allclose(res["scores"][i, sel], sc[r][idx[i, sel]], rtol=1e-12,
                                   atol=1e-14)
        ref = entropy(target[i, sel], softmax(sc[r][idx[i, sel]]))
        assert res["loss"][i] == pytest.approx(ref, rel=1e-10, abs=1e-14)


def _random_real_case(seed, n=2, h=3, d=5, k=7):
    """Real-valued inputs whose dot products stay away from the ReLU kink."""
    g = np.random.default_rng(seed)
    while True:
        q = g.standard_normal((n, h, d))
        keys = g.standard_normal((n, k, d))
        if np.abs(np.einsum("rjd,red->rje", q, keys)).min() > 0.05:
            break
    w = g.uniform(0.2, 1.5, (n, h))
    valid = np.ones((n, k), np.int32)
    valid[0, 2] = 0
    target = g.uniform(0.1, 1.0, (n, k)) * valid
    target[0] /= target[0].sum()
    target[1] *= 0.7 / target[1].sum()                  # a target that does not sum to 1
    return q, w, keys, valid, target


def test_indexer_kl_gradients_match_finite_differences():
    q, w, keys, valid, target = _random_real_case(11)
    res = oracle.indexer_kl_real(q, w, keys, valid, target)
    f = lambda q_, w_, k_: oracle.indexer_kl_real(q_, w_, k_, valid, target)["loss"].sum()
    eps = 1e-6
    for name, arr, grad in (("q", q, res["dq"]), ("w", w, res["dw"]), ("keys", keys, res["dk"])):
        num = np.zeros_like(arr)
        for ix in np.ndindex(arr.shape):
            a, b = arr.copy(), arr.copy()
            a[ix] += eps
            b[ix] -= eps
            args = {"q": (q, w, keys), "w": (q, w, keys), "keys": (q, w, keys)}[name]
            fa = f(*(a if x is arr else x for x in args))
            fb = f(*(b if x is arr else x for x in args))
            num[ix] = (fa - fb) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8, err_msg=name)
    assert not res["dk"][0, 2].any()                    # unused slot: no gradient


def test_indexer_kl_vanishes_when_the_target_is_the_indexer_distribution():
    from scipy.special import softmax
    q, w, keys, valid, _ = _random_real_case(12)
    s = np.maximum(np.einsum("rjd,red->rje", q, keys), 0.0)
    scores = np.einsum("rj,rje->re", w, s)
    target = np.where(valid > 0, softmax(np.where(valid > 0, scores, -np.inf), axis=1), 0.0)
    res = oracle.indexer_kl_real(q, w, keys, valid, target)
    assert np.abs(res["loss"]).max() < 1e-14
    for key in ("dq", "dw", "dk"):
        assert np.abs(res[key]).max() < 1e-13, key


def test_indexer_kl_key_gradient_sums_over_rows():
    """A physical key selected by several rows receives the sum of their gradients."""
    wl = _kl_workload()
    rows = [40, 41, 59]
    _, idx, _, _ = oracle.forward_rows(wl, rows)
    target = oracle.kl_target_rows(wl, rows, idx)
    both = oracle.indexer_kl_rows(wl, rows, idx, target)
    acc = {}
    for i, r in enumerate(rows):
        one = oracle.indexer_kl_rows(wl, [r], idx[i:i + 1], target[i:i + 1])
        for p, g in zip(one["dk_rows"], one["dk"]):
            acc[int(p)] = acc.get(int(p), 0.0) + g
    assert sorted(acc) == both["dk_rows"].tolist()
    for p, g in zip(both["dk_rows"], both["dk"]):
        np.testing.assert_allclose(g, acc[int(p)], rtol=1e-12, atol=1e-15)


def test_training_oracle_matches_numpy_twin():
    """The C oracle's target and KL gradients equal the independent NumPy twin's."""
    wl = _tiny_attn_workload()
    rows = [30, 39]
    idx = np.array([[3, 11, 0, -1, 25, 7, 30, -1], [39, 38, 37, 4, -1, -1, -1, -1]], np.int32)
    t = oracle.kl_target_rows(wl, rows, idx)
    qb = wl.q.view(torch.int16).numpy().view(np.uint16)
    kvb = wl.kv.view(torch.int16).numpy().view(np.uint16)
    for i, r in enumerate(rows):   # a single prefill sequence: logical key s is physical row s
        np.testing.assert_allclose(t[i], reference_np.kl_target(qb[r], kvb, idx[i], 0.3),
                                   rtol=1e-12, atol=1e-15)
    q, w, keys, valid, target = _random_real_case(13, n=3, h=4, d=6, k=9)
    res = oracle.indexer_kl_real(q, w, keys, valid, target)
    for i in range(3):
        loss, dw, dq, dk = reference_np.indexer_kl(q[i], w[i], keys[i], valid[i] > 0, target[i])
        assert res["loss"][i] == pytest.approx(loss, rel=1e-12, abs=1e-15)
        np.testing.assert_allclose(res["dw"][i], dw, rtol=1e-11, atol=1e-14)
        np.testing.assert_allclose(res["dq"][i], dq, rtol=1e-11, atol=1e-14)
        np.testing.assert_allclose(res["dk"][i], dk, rtol=1e-11, atol=1e-14)
