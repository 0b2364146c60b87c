"""C-ABI checks that need no GPU: the library loads, exports every entry point that
include/dsa.h declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def dsa():
    import importlib.util
    # build.py by path: importing the package first would load a stale library
    spec = importlib.util.spec_from_file_location(
        "_dsa_lib_build", os.path.join(ROOT, "sparse_attention_long_04_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    import sparse_attention_long_04_b200 as m
    return m


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    return sorted(set(re.findall(r"^DSA_API\s+[\w\s\*]+?\b(dsa_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for n in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_fwd", "dsa_forward",
              "dsa_forward_workspace_size", "dsa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(dsa):
    lib = ctypes.CDLL(dsa.LIB_PATH)
    for n in declared_symbols():
        assert hasattr(lib, n), n
    assert set(dsa.EXPORTED) >= set(declared_symbols())
    assert dsa.abi_version() == 3
    assert dsa.status_string(0) == "ok"
    assert "workspace" in dsa.status_string(3)


FAKE = 0x10000   # a 16-byte-aligned address that is never dereferenced: validation fails first


def _pb(dsa, **kw):
    args = dict(mode="decode", h_idx=64, d_idx=128, h=128, d_qk=576, d_v=512, topk=2048,
                softmax_scale=0.04, num_kv_rows=1 << 20, seqlens=[4096, 100],
                seq_lens=FAKE, block_table=None, max_seqlen=4096)
    args.update(kw)
    pb = dsa.make_problem(**{k: v for k, v in args.items() if k != "seq_lens"},
                          seq_lens=None)
    pb.seqs.seq_lens = args["seq_lens"]
    return pb


def test_null_pointers_rejected(dsa):
    pb = _pb(dsa)
    st = dsa.dsa_indexer_scores(pb, None, FAKE, FAKE, FAKE, FAKE, 0, 2, FAKE, 4096, None, 0)
    assert st == dsa.DSA_ERR_INVALID_ARG
    st = dsa.dsa_topk(pb, FAKE, 4096, 0, 2, None, None, 0)
    assert st == dsa.DSA_ERR_INVALID_ARG
    st = dsa.dsa_sparse_mla_fwd(pb, FAKE, FAKE, FAKE, 0, 2, FAKE, None, None, 0, None, 0)
    assert st == dsa.DSA_ERR_INVALID_ARG
    lib = dsa.lib
    assert lib.dsa_forward(None, None, *([None] * 12), 0, None, None) == dsa.DSA_ERR_INVALID_ARG


def test_bad_shapes_rejected(dsa):
    assert dsa.dsa_indexer_scores(_pb(dsa, h_idx=32), FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, FAKE,
                                  4096, None, 0) == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    assert dsa.dsa_sparse_mla_fwd(_pb(dsa, d_qk=512), FAKE, FAKE, FAKE, 0, 2, FAKE, FAKE, None,
                                  0, None, 0) == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    assert dsa.dsa_topk(_pb(dsa, topk=100), FAKE, 4096, 0, 2, FAKE, None,
                        0) == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    # the tiny indexer shape is prefill-only
    assert dsa.dsa_indexer_scores(_pb(dsa, h_idx=4, d_idx=32), FAKE, FAKE, FAKE, FAKE, FAKE, 0,
                                  2, FAKE, 4096, None, 0) == dsa.DSA_ERR_UNSUPPORTED_SHAPE


def test_misaligned_and_bad_ld_rejected(dsa):
    pb = _pb(dsa)
    assert dsa.dsa_indexer_scores(pb, FAKE + 8, FAKE, FAKE, FAKE, FAKE, 0, 2, FAKE, 4096, None,
                                  0) == dsa.DSA_ERR_MISALIGNED
    assert dsa.dsa_topk(pb, FAKE, 4098, 0, 2, FAKE, None, 0) == dsa.DSA_ERR_MISALIGNED
    assert dsa.dsa_sparse_mla_fwd(pb, FAKE, FAKE + 4, FAKE, 0, 2, FAKE, FAKE, None, 0, None,
                                  0) == dsa.DSA_ERR_MISALIGNED
    # ld below the longest row
    assert dsa.dsa_topk(pb, FAKE, 1024, 0, 2, FAKE, None, 0) == dsa.DSA_ERR_INVALID_ARG


def test_bad_geometry_rejected(dsa):
    pb = _pb(dsa)
    assert dsa.dsa_topk(pb, FAKE, 4096, 1, 2, FAKE, None, 0) == dsa.DSA_ERR_INVALID_ARG  # rows
    pre = dsa.make_problem(mode="prefill", h_idx=64, d_idx=128, h=128, d_qk=576, d_v=512,
                           topk=2048, softmax_scale=0.04, num_kv_rows=100, seqlens=[60, 70],
                           cu_seqlens=FAKE)
    # more packed rows than cache rows
    assert dsa.dsa_topk(pre, FAKE, 72, 0, 130, FAKE, None, 0) == dsa.DSA_ERR_INVALID_ARG
    pre.seqs.cu_seqlens_host = None
    assert dsa.dsa_topk(pre, FAKE, 72, 0, 1, FAKE, None, 0) == dsa.DSA_ERR_INVALID_ARG
    # a block table narrower than the longest sequence
    pb2 = _pb(dsa)
    pb2.seqs.block_table = FAKE
    pb2.seqs.max_blocks = 10
    assert dsa.dsa_topk(pb2, FAKE, 4096, 0, 2, FAKE, None, 0) == dsa.DSA_ERR_INVALID_ARG


def test_workspace_size_is_zero_on_bad_args(dsa):
    pb = _pb(dsa, topk=7)
    assert dsa.dsa_forward_workspace_size(pb) == 0


def test_cache_append_argument_errors(dsa):
    """The append is decode-only, needs its five buffers and 16-byte alignment, and supports
    the two key/latent widths; all of this is rejected before any launch."""
    pb = _pb(dsa)
    ok = [FAKE] * 5
    call = lambda p, bufs: dsa.dsa_cache_append(p, *bufs, None, 0)
    assert call(pb, [None] + ok[1:]) == dsa.DSA_ERR_INVALID_ARG
    assert call(pb, [FAKE + 4] + ok[1:]) == dsa.DSA_ERR_MISALIGNED
    pre = dsa.make_problem(mode="prefill", h_idx=64, d_idx=128, h=128, d_qk=576, d_v=512,
                           topk=2048, softmax_scale=0.04, num_kv_rows=1 << 20, seqlens=[100],
                           cu_seqlens=FAKE)
    assert call(pre, ok) == dsa.DSA_ERR_INVALID_ARG
    odd = _pb(dsa, d_qk=512)
    assert call(odd, ok) == dsa.DSA_ERR_UNSUPPORTED_SHAPE


def test_dense_attention_row_rules(dsa):
    """Attention without an index array means every prior key.  Prefill rows may be of any
    length (dense causal attention); a decode batch whose contexts exceed topk, and the training
    target without indices over a row of more than topk keys (it writes topk entries per row),
    are refused before any launch; the dense warm-up calls check their row strides."""
    pre = dsa.make_problem(mode="prefill", h_idx=64, d_idx=128, h=128, d_qk=576, d_v=512,
                           topk=2048, softmax_scale=0.04, num_kv_rows=1 << 20,
                           seqlens=[5000], cu_seqlens=FAKE)
    dec = _pb(dsa, max_seqlen=4096)
    assert dsa.dsa_sparse_mla_fwd(dec, FAKE, FAKE, None, 0, 2, FAKE, FAKE, None, 0, None,
                                  0) == dsa.DSA_ERR_INVALID_ARG
    # rows 0..2047 have at most 2048 prior keys; row 2048 has 2049
    assert dsa.dsa_indexer_kl_target(pre, FAKE, FAKE, None, FAKE, 2000, 100, FAKE, None,
                                     0) == dsa.DSA_ERR_INVALID_ARG
    tgt = dsa.dsa_indexer_kl_target_dense
    assert tgt(pre, FAKE, FAKE, FAKE, 2000, 100, FAKE, 2048, None, 0) == dsa.DSA_ERR_INVALID_ARG
    assert tgt(pre, FAKE, FAKE, FAKE, 2000, 100, FAKE, 2110, None, 0) == dsa.DSA_ERR_MISALIGNED
    assert tgt(dec, FAKE, FAKE, FAKE, 0, 2, FAKE, 4096, None, 0) == dsa.DSA_ERR_INVALID_ARG
    bwd = dsa.dsa_indexer_kl_backward_dense
    f = [FAKE] * 5
    out = [FAKE] * 4
    assert bwd(pre, *f, FAKE, 2048, 2000, 100, *out, None, 0) == dsa.DSA_ERR_INVALID_ARG
    assert bwd(pre, *f, FAKE, 2102, 2000, 100, *out, None, 0) == dsa.DSA_ERR_MISALIGNED
    assert bwd(dec, *f, FAKE, 4096, 0, 2, *out, None, 0) == dsa.DSA_ERR_INVALID_ARG
    assert dsa.dsa_indexer_kl_backward(pre, *f, None, FAKE, 0, 2, *out, None,
                                       0) == dsa.DSA_ERR_INVALID_ARG


def test_scales_inside_key_blocks_only_for_paged_decode(dsa):
    """k_scale NULL (scales stored inside the 64-row key blocks) is accepted only for paged
    decode; elsewhere it is an argument error."""
    dec = _pb(dsa)                                     # decode without a block table
    assert dsa.dsa_indexer_scores(dec, FAKE, FAKE, FAKE, FAKE, None, 0, 2, FAKE, 4096, None,
                                  0) == dsa.DSA_ERR_INVALID_ARG
    assert dsa.dsa_cache_append(dec, FAKE, FAKE, FAKE, None, FAKE, None,
                                0) == dsa.DSA_ERR_INVALID_ARG


def test_wait_selftest_argument_errors(dsa):
    """The bounded-wait self-test needs a 4-byte-aligned status word; both are checked before
    any launch."""
    assert dsa.dsa_selftest_wait_timeout(None, 0) == dsa.DSA_ERR_INVALID_ARG
    assert dsa.dsa_selftest_wait_timeout(FAKE + 2, 0) == dsa.DSA_ERR_MISALIGNED


def test_probe_argument_errors(dsa):
    """The two diagnostics check counts, sizes and alignment before any launch."""
    lib, INV, MIS = dsa.lib, dsa.DSA_ERR_INVALID_ARG, dsa.DSA_ERR_MISALIGNED
    ok = dict(base=FAKE, ids=FAKE, n_ids=4, n_blocks=4, d_idx=128, cps=2, bad=FAKE)

    def stream(**kw):
        a = dict(ok, **kw)
        return lib.dsa_probe_page_stream(a["base"], a["ids"], a["n_ids"], a["n_blocks"],
                                         a["d_idx"], a["cps"], a["bad"], 0)

    for kw in (dict(base=None), dict(ids=None), dict(bad=None), dict(n_ids=0),
               dict(n_blocks=0), dict(n_blocks=1 << 31), dict(d_idx=0), dict(d_idx=64),
               dict(cps=0), dict(cps=9)):
        assert stream(**kw) == INV, kw
    for kw in (dict(base=FAKE + 8), dict(ids=FAKE + 2), dict(bad=FAKE + 2)):
        assert stream(**kw) == MIS, kw
    assert lib.dsa_probe_dsmem(0, 32768, 4, FAKE, FAKE, 0) == INV
    assert lib.dsa_probe_dsmem(1, 100, 4, FAKE, FAKE, 0) == INV
    assert lib.dsa_probe_dsmem(1, 32768, 0, FAKE, FAKE, 0) == INV
    assert lib.dsa_probe_dsmem(1, 32768, 4, FAKE + 4, FAKE, 0) == MIS


def test_indexer_training_argument_errors(dsa):
    """The target and backward calls check their pointers, alignment, shapes and rows before
    any launch."""
    pb = _pb(dsa)

    def target(p, q=FAKE, kv=FAKE, idx=FAKE, lse=FAKE, tgt=FAKE, rb=0, n=2):
        return dsa.dsa_indexer_kl_target(p, q, kv, idx, lse, rb, n, tgt, None, 0)

    assert target(pb, lse=None) == dsa.DSA_ERR_INVALID_ARG
    assert target(pb, idx=None) == dsa.DSA_ERR_INVALID_ARG     # rows longer than topk
    assert target(pb, tgt=FAKE + 4) == dsa.DSA_ERR_MISALIGNED
    assert target(pb, rb=1) == dsa.DSA_ERR_INVALID_ARG          # past the last row
    assert target(_pb(dsa, d_qk=512)) == dsa.DSA_ERR_UNSUPPORTED_SHAPE

    ok = [FAKE] * 11   # q_idx, q_scale, w, k_idx, k_scale, idx, target | loss, dw, dq, dk

    def backward(p, bufs, rb=0, n=2):
        return dsa.dsa_indexer_kl_backward(p, *bufs[:7], rb, n, *bufs[7:], None, 0)

    assert backward(pb, ok[:4] + [None] + ok[5:]) == dsa.DSA_ERR_INVALID_ARG   # k_scale
    assert backward(pb, ok[:5] + [None] + ok[6:]) == dsa.DSA_ERR_INVALID_ARG   # idx
    assert backward(pb, ok[:10] + [None]) == dsa.DSA_ERR_INVALID_ARG          # dk
    assert backward(pb, [FAKE + 4] + ok[1:]) == dsa.DSA_ERR_MISALIGNED
    assert backward(pb, ok, rb=1) == dsa.DSA_ERR_INVALID_ARG
    assert backward(_pb(dsa, h_idx=32), ok) == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    # the tensor-core kernel of the 64 x 128 indexer takes the selection in 128-key tiles
    assert backward(_pb(dsa, topk=192), ok) == dsa.DSA_ERR_UNSUPPORTED_SHAPE


def test_forward_workspace_plan_on_the_host(dsa):
    """Workspace sizes of `dsa_forward` for a given SM count, with no device involved.  A decode
    batch needs a score slab of every sequence's padded row and its indices; a prefill sequence
    is cut into chunks of at most 256 MiB of fp32 scores, and a sequence that needs several
    chunks gets a multiple of sm_count / 2 rows per chunk (whole waves of two-CTA rows)."""
    full = dict(h_idx=64, d_idx=128, h=128, d_qk=576, d_v=512, topk=2048, softmax_scale=0.04)
    size = dsa.dsa_forward_workspace_size_for
    # decode_B64_N128k shapes, contiguous caches: 128 attention CTAs fill one wave of 148 SMs,
    # so no split-KV partials
    # (+ the fused indexer's first-digit histograms: 2048 words per row of a chunk)
    H = 2048 * 4
    dec = dsa.make_problem(mode="decode", num_kv_rows=64 * 131072, seqlens=[131072] * 64,
                           seq_lens=FAKE, max_seqlen=131072, **full)
    assert size(dec, 148) == 64 * 131072 * 4 + 64 * 2048 * 4 + 64 * H
    # a few long decode rows on many SMs are split, and the partials add to the workspace
    few = dsa.make_problem(mode="decode", num_kv_rows=2 * 131072, seqlens=[131072] * 2,
                           seq_lens=FAKE, max_seqlen=131072, **full)
    assert size(few, 148) > 2 * 131072 * 4 + 2 * 2048 * 4 + 2 * H
    # prefill: 131072 rows need 512 rows of scores per 256 MiB; 148 SMs -> 444 (6 x 74) rows
    pre = dsa.make_problem(mode="prefill", num_kv_rows=131072, seqlens=[131072],
                           cu_seqlens=FAKE, **full)
    assert size(pre, 148) == 444 * 131072 * 4 + 444 * 2048 * 4 + 444 * H
    assert size(pre, 132) == 462 * 131072 * 4 + 462 * 2048 * 4 + 462 * H   # 7 x 66 rows
    # a short sequence runs in one chunk; varlen sizes the slab for the largest chunk's scores
    # and the indices for the chunk with the most rows (here the short sequence's 1000)
    short = dsa.make_problem(mode="prefill", num_kv_rows=1000, seqlens=[1000], cu_seqlens=FAKE,
                             **full)
    assert size(short, 148) == 1000 * 1000 * 4 + 1000 * 2048 * 4 + 1000 * H
    mix = dsa.make_problem(mode="prefill", num_kv_rows=132072, seqlens=[1000, 131072],
                           cu_seqlens=FAKE, **full)
    assert size(mix, 148) == 444 * 131072 * 4 + 1000 * 2048 * 4 + 1000 * H
    # the small indexer shape builds its histograms in the top-k: none in the workspace
    tiny = dsa.make_problem(mode="prefill", num_kv_rows=1024, seqlens=[1024], cu_seqlens=FAKE,
                            h_idx=4, d_idx=32, h=16, d_qk=160, d_v=128, topk=64,
                            softmax_scale=0.08)
    assert size(tiny, 148) == 1024 * 1024 * 4 + 1024 * 64 * 4
    assert size(pre, 0) == 0 and size(_pb(dsa, topk=100), 148) == 0
    # the chunk plan itself: rows per chunk of each sequence
    rows = dsa.dsa_forward_chunk_rows_for
    assert rows(pre, 0, 148) == 444 and rows(pre, 0, 132) == 462
    assert rows(mix, 0, 148) == 1000 and rows(mix, 1, 148) == 444
    assert rows(mix, 2, 148) == 0 and rows(dec, 0, 148) == 64


def test_noalloc_partials_fit_the_builtin_array_for_every_batch(dsa):
    """The allocation-free attention entry point sizes its split-KV partials to its built-in
    array: for every decode batch of 1..4096 rows at full shapes, on 148 and 132 SMs, the capped
    choice fits DSA_NOALLOC_SCRATCH_BYTES, equals the uncapped choice whenever that one fits,
    and falls back to no partials at all otherwise."""
    full = dict(h_idx=64, d_idx=128, h=128, d_qk=576, d_v=512, topk=2048, softmax_scale=0.04)
    cap = dsa.NOALLOC_SCRATCH_BYTES
    per_split_row = 128 * 513 * 4
    for sms in (148, 132):
        for rows in range(1, 4097):
            pb = dsa.make_problem(mode="decode", num_kv_rows=rows * 8192, seqlens=[8192] * rows,
                                  seq_lens=FAKE, max_seqlen=8192, **full)
            free = dsa.dsa_sparse_mla_workspace_size_for(pb, rows, sms)
            capped = dsa.dsa_sparse_mla_workspace_size_for(pb, rows, sms, cap)
            assert capped <= cap, (sms, rows, capped)
            if free <= cap:
                assert capped == free, (sms, rows)
            assert capped == 0 or (capped - 256) % (rows * per_split_row) == 0
    # the bound at full shapes: splits * rows * 128 * 513 * 4 + 256 <= 20 MiB -> <= 79 row-splits
    assert (cap - 256) // per_split_row == 79


def test_fused_indexer_topk_arguments(dsa):
    """dsa_indexer_topk: workspace sizing on the host (slab of the rows at max_seqlen keys plus
    2048 histogram words per row) and argument errors before any launch."""
    pb = _pb(dsa)
    need = dsa.dsa_indexer_topk_workspace_size(pb, 2)
    assert need == 2 * 4096 * 4 + 2 * 2048 * 4
    args = [FAKE, FAKE, FAKE, FAKE, FAKE]        # q_idx, q_scale, w, k_idx, k_scale

    def call(p, a, rb=0, n=2, idx=FAKE, ws=FAKE, wsb=None):
        return dsa.dsa_indexer_topk(p, *a, rb, n, idx, ws, need if wsb is None else wsb, None, 0)

    assert call(pb, args, idx=None) == dsa.DSA_ERR_INVALID_ARG
    assert call(pb, [None] + args[1:]) == dsa.DSA_ERR_INVALID_ARG
    assert call(pb, args, wsb=need - 1) == dsa.DSA_ERR_WORKSPACE_TOO_SMALL
    assert call(pb, args, ws=None) == dsa.DSA_ERR_WORKSPACE_TOO_SMALL
    assert call(pb, args, ws=FAKE + 8) == dsa.DSA_ERR_MISALIGNED
    assert call(pb, args, rb=1) == dsa.DSA_ERR_INVALID_ARG
    assert call(_pb(dsa, h_idx=32), args) == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    assert call(pb, args, n=0) == dsa.DSA_OK        # nothing to do, nothing launched


def test_stage_histogram_arguments(dsa):
    """The optional first-digit histograms of dsa_indexer_scores / dsa_topk: 16-byte alignment,
    and only the 64 x 128 indexer counts them."""
    pb = _pb(dsa)
    st = dsa.dsa_indexer_scores(pb, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, FAKE, 4096, None, 0,
                                hist=FAKE + 4)
    assert st == dsa.DSA_ERR_MISALIGNED
    st = dsa.dsa_topk(pb, FAKE, 4096, 0, 2, FAKE, None, 0, hist=FAKE + 4)
    assert st == dsa.DSA_ERR_MISALIGNED
    tiny = dsa.make_problem(mode="prefill", num_kv_rows=1024, seqlens=[1024], cu_seqlens=FAKE,
                            h_idx=4, d_idx=32, h=16, d_qk=160, d_v=128, topk=64,
                            softmax_scale=0.08)
    st = dsa.dsa_indexer_scores(tiny, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, FAKE, 1024, None, 0,
                                hist=FAKE)
    assert st == dsa.DSA_ERR_UNSUPPORTED_SHAPE


def test_selected_scores_arguments(dsa):
    """The optional scores of the selected keys (sel_out of the selection and the forward,
    sel_scores of the KL backward): 16-byte alignment, and the forward keeps them only with the
    indices."""
    pb = _pb(dsa)
    assert dsa.dsa_topk(pb, FAKE, 4096, 0, 2, FAKE, None, 0,
                        sel_out=FAKE + 4) == dsa.DSA_ERR_MISALIGNED
    need = dsa.dsa_indexer_topk_workspace_size(pb, 2)
    assert dsa.dsa_indexer_topk(pb, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, FAKE, FAKE, need, None, 0,
                                sel_out=FAKE + 8) == dsa.DSA_ERR_MISALIGNED
    # q_idx, q_scale, w, k_idx, k_scale, q, kv, idx_out = None, out, lse, workspace, sel_out
    st = dsa.dsa_forward(pb, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE,
                         1 << 30, None, 0, sel_out=FAKE)
    assert st == dsa.DSA_ERR_INVALID_ARG
    st = dsa.dsa_forward_rows(pb, 0, 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                              FAKE, FAKE, 1 << 30, None, 0, sel_out=FAKE)
    assert st == dsa.DSA_ERR_INVALID_ARG
    out = [FAKE] * 4                              # loss, dw, dq, dk
    st = dsa.dsa_indexer_kl_backward(pb, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, *out,
                                     None, 0, sel=FAKE + 4)
    assert st == dsa.DSA_ERR_MISALIGNED
