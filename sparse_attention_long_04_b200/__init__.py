"""B200 (sm_100a) DeepSeek Sparse Attention hot path: Python binding of ``libdsa.so``.

The library (``include/dsa.h``) runs the three DSA stages in hand-written CUDA kernels:
the FP8 lightning indexer, the exact top-k selector and sparse MLA attention in MQA mode
("FP8 index -> top-k selection -> sparse core attention", "DeepSeek V3.2-Exp Cuts
Long-Context Costs with DeepSeek Sparse Attention (DSA)", pipeline summary), plus the decode
cache append and the indexer's training step (KL target and backward, same page, "Training
signal").

This module only marshals arguments: the functions named like the C entry points take torch
tensors (device memory owned by the caller), pass their pointers and the current CUDA stream,
and return the integer status.  Nothing is computed here, and there is no fallback: importing
fails if the built library is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libdsa.so")

DSA_OK = 0
DSA_ERR_INVALID_ARG = 1
DSA_ERR_UNSUPPORTED_SHAPE = 2
DSA_ERR_WORKSPACE_TOO_SMALL = 3
DSA_ERR_MISALIGNED = 4
DSA_ERR_BAD_INDEX = 5
DSA_ERR_TIMEOUT = 6
DSA_ERR_CUDA = 7
DSA_DEVICE_TIMEOUT = 1
DSA_DEVICE_BAD_INDEX = 2
TOPK_HIST_BINS = 2048
DSA_PREFILL = 0
DSA_DECODE = 1

EXPORTED = ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_workspace_size",
            "dsa_sparse_mla_fwd", "dsa_forward_workspace_size", "dsa_forward",
            "dsa_read_device_status", "dsa_status_string", "dsa_abi_version",
            "dsa_sparse_mla_fwd_noalloc", "dsa_cache_append", "dsa_selftest_wait_timeout",
            "dsa_indexer_kl_target", "dsa_indexer_kl_backward", "dsa_forward_workspace_size_for",
            "dsa_sparse_mla_workspace_size_for", "dsa_indexer_topk",
            "dsa_indexer_topk_workspace_size", "dsa_forward_chunk_rows_for",
            "dsa_forward_rows", "dsa_indexer_kl_target_dense", "dsa_indexer_kl_backward_dense",
            "dsa_probe_dsmem", "dsa_probe_page_stream")
NOALLOC_SCRATCH_BYTES = 20 << 20


class DsaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})" if what else
                         f"{status_string(status)} ({status})")


class dsa_dims_t(ctypes.Structure):
    _fields_ = [("h_idx", ctypes.c_int32), ("d_idx", ctypes.c_int32), ("h", ctypes.c_int32),
                ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("softmax_scale", ctypes.c_float)]


class dsa_seqs_t(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("total_rows", ctypes.c_int32), ("max_seqlen", ctypes.c_int32),
                ("num_kv_rows", ctypes.c_int64), ("cu_seqlens", ctypes.c_void_p),
                ("cu_seqlens_host", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("max_blocks", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libdsa.so is not built ({LIB_PATH}); run "
                          "`python -c 'import __graft_entry__ as g; g.build()'` or "
                          "`python sparse_attention_long_04_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    DP, SP = ctypes.POINTER(dsa_dims_t), ctypes.POINTER(dsa_seqs_t)
    sig = {
        "dsa_indexer_scores": (I32, [DP, SP, P, P, P, P, P, I32, I32, P, I64, P, P, P]),
        "dsa_topk": (I32, [DP, SP, P, I64, P, I32, I32, P, P, P, P]),
        "dsa_indexer_topk_workspace_size": (SZ, [DP, SP, I32]),
        "dsa_indexer_topk": (I32, [DP, SP, P, P, P, P, P, I32, I32, P, P, P, SZ, P, P]),
        "dsa_sparse_mla_workspace_size": (SZ, [DP, SP, I32]),
        "dsa_sparse_mla_fwd": (I32, [DP, SP, P, P, P, I32, I32, P, P, P, SZ, P, P]),
        "dsa_forward_workspace_size": (SZ, [DP, SP]),
        "dsa_forward_workspace_size_for": (SZ, [DP, SP, I32]),
        "dsa_forward_chunk_rows_for": (I32, [DP, SP, I32, I32]),
        "dsa_sparse_mla_workspace_size_for": (SZ, [DP, SP, I32, I32, SZ]),
        "dsa_forward": (I32, [DP, SP, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P, P]),
        "dsa_forward_rows": (I32, [DP, SP, I32, I32, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P,
                                   P]),
        "dsa_read_device_status": (I32, [P, P, ctypes.POINTER(ctypes.c_int32)]),
        "dsa_selftest_wait_timeout": (I32, [P, P]),
        "dsa_probe_dsmem": (I32, [I32, I32, I32, P, P, P]),
        "dsa_probe_page_stream": (I32, [P, P, I64, I64, I32, I32, P, P]),
        "dsa_indexer_kl_target": (I32, [DP, SP, P, P, P, P, I32, I32, P, P, P]),
        "dsa_indexer_kl_target_dense": (I32, [DP, SP, P, P, P, I32, I32, P, I64, P, P]),
        "dsa_indexer_kl_backward_dense": (I32, [DP, SP, P, P, P, P, P, P, I64, I32, I32, P, P, P,
                                                P, P, P]),
        "dsa_indexer_kl_backward": (I32, [DP, SP, P, P, P, P, P, P, P, P, I32, I32, P, P, P, P,
                                          P, P]),
        "dsa_status_string": (ctypes.c_char_p, [I32]),
        "dsa_abi_version": (I32, []),
        "dsa_sparse_mla_fwd_noalloc": (I32, [DP, SP, P, P, P, I32, I32, P, P, P, P]),
        "dsa_cache_append": (I32, [DP, SP, P, P, P, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


lib = _load()


def status_string(status: int) -> str:
    return lib.dsa_status_string(int(status)).decode()


def abi_version() -> int:
    return int(lib.dsa_abi_version())


# ---------------------------------------------------------------------- marshalling helpers

def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class Problem:
    """The dims and sequence structs of one DSA call, plus the host arrays they point to."""

    def __init__(self, dims: dsa_dims_t, seqs: dsa_seqs_t, keep=()):
        self.dims = dims
        self.seqs = seqs
        self._keep = list(keep)


def make_problem(*, mode: str, h_idx: int, d_idx: int, h: int, d_qk: int, d_v: int, topk: int,
                 softmax_scale: float, num_kv_rows: int, seqlens, cu_seqlens=None,
                 seq_lens=None, block_table=None, max_seqlen: Optional[int] = None,
                 block_size: int = 64) -> Problem:
    """Builds dsa_dims_t / dsa_seqs_t.  ``cu_seqlens``, ``seq_lens``, ``block_table`` are device
    int32 tensors; ``seqlens`` is the host list of sequence lengths."""
    dims = dsa_dims_t(h_idx, d_idx, h, d_qk, d_v, topk, block_size, softmax_scale)
    seqlens = [int(x) for x in seqlens]
    max_len = int(max_seqlen or max(seqlens))
    keep = []
    s = dsa_seqs_t()
    s.batch = len(seqlens)
    s.max_seqlen = max_len
    s.num_kv_rows = int(num_kv_rows)
    if mode == "prefill":
        host = (ctypes.c_int32 * (len(seqlens) + 1))()
        acc = 0
        for i, L in enumerate(seqlens):
            host[i] = acc
            acc += L
        host[len(seqlens)] = acc
        keep.append(host)
        s.mode = DSA_PREFILL
        s.total_rows = acc
        s.cu_seqlens = _ptr(cu_seqlens)
        s.cu_seqlens_host = ctypes.cast(host, ctypes.c_void_p)
    else:
        s.mode = DSA_DECODE
        s.total_rows = len(seqlens)
        s.seq_lens = _ptr(seq_lens)
        s.block_table = _ptr(block_table)
        s.max_blocks = int(block_table.shape[1]) if block_table is not None else 0
    keep.extend(t for t in (cu_seqlens, seq_lens, block_table) if t is not None)
    return Problem(dims, s, keep)


def problem_of(wl) -> Problem:
    """Problem for a workload object (``dsa_workloads.Workload`` or any object with the same
    attributes)."""
    d = wl.dims
    return make_problem(mode=wl.mode, h_idx=d["h_idx"], d_idx=d["d_idx"], h=d["h"],
                        d_qk=d["d_qk"], d_v=d["d_v"], topk=d["topk"],
                        softmax_scale=float(wl.softmax_scale), num_kv_rows=wl.kv.shape[0],
                        seqlens=wl.seqlens, cu_seqlens=wl.cu_seqlens, seq_lens=wl.seq_lens,
                        block_table=wl.block_table, max_seqlen=wl.max_seqlen)


# ---------------------------------------------------------------------- the C entry points

def dsa_indexer_scores(pb: Problem, q_idx, q_scale, w, k_idx, k_scale, row_begin: int,
                       row_count: int, scores, ld_scores: int, dev_status=None,
                       stream=None, hist=None) -> int:
    return int(lib.dsa_indexer_scores(
        ctypes.byref(pb.dims), ctypes.byref(pb.seqs), _ptr(q_idx), _ptr(q_scale), _ptr(w),
        _ptr(k_idx), _ptr(k_scale), row_begin, row_count, _ptr(scores), ld_scores, _ptr(hist),
        _ptr(dev_status), _stream(stream)))


def dsa_topk(pb: Problem, scores, ld_scores: int, row_begin: int, row_count: int, idx,
             dev_status=None, stream=None, hist=None, sel_out=None) -> int:
    return int(lib.dsa_topk(ctypes.byref(pb.dims), ctypes.byref(pb.seqs), _ptr(scores),
                            ld_scores, _ptr(hist), row_begin, row_count, _ptr(idx),
                            _ptr(sel_out), _ptr(dev_status), _stream(stream)))


def dsa_indexer_topk_workspace_size(pb: Problem, row_count: int) -> int:
    return int(lib.dsa_indexer_topk_workspace_size(ctypes.byref(pb.dims), ctypes.byref(pb.seqs),
                                                   row_count))


def dsa_indexer_topk(pb: Problem, q_idx, q_scale, w, k_idx, k_scale, row_begin: int,
                     row_count: int, idx, workspace, workspace_bytes: int, dev_status=None,
                     stream=None, sel_out=None) -> int:
    return int(lib.dsa_indexer_topk(
        ctypes.byref(pb.dims), ctypes.byref(pb.seqs), _ptr(q_idx), _ptr(q_scale), _ptr(w),
        _ptr(k_idx), _ptr(k_scale), row_begin, row_count, _ptr(idx), _ptr(sel_out),
        _ptr(workspace), workspace_bytes, _ptr(dev_status), _stream(stream)))


def dsa_sparse_mla_workspace_size(pb: Problem, row_count: int) -> int:
    return int(lib.dsa_sparse_mla_workspace_size(ctypes.byref(pb.dims), ctypes.byref(pb.seqs),
                                                 row_count))


def dsa_sparse_mla_workspace_size_for(pb: Problem, row_count: int, sm_count: int,
                                      max_bytes: Optional[int] = None) -> int:
    """Host-only sizing (no device needed); max_bytes None = no cap."""
    cap = ctypes.c_size_t(-1).value if max_bytes is None else int(max_bytes)
    return int(lib.dsa_sparse_mla_workspace_size_for(ctypes.byref(pb.dims),
                                                     ctypes.byref(pb.seqs), row_count,
                                                     sm_count, cap))


def dsa_sparse_mla_fwd(pb: Problem, q, kv, idx, row_begin: int, row_count: int, out, lse,
                       workspace=None, workspace_bytes: int = 0, dev_status=None,
                       stream=None) -> int:
    return int(lib.dsa_sparse_mla_fwd(
        ctypes.byref(pb.dims), ctypes.byref(pb.seqs), _ptr(q), _ptr(kv), _ptr(idx), row_begin,
        row_count, _ptr(out), _ptr(lse), _ptr(workspace), workspace_bytes, _ptr(dev_status),
        _stream(stream)))


def dsa_sparse_mla_fwd_noalloc(pb: Problem, q, kv, idx, row_begin: int, row_count: int, out, lse,
                               dev_status=None, stream=None) -> int:
    """dsa_sparse_mla_fwd without a workspace, for callers that may not allocate device memory
    (its scratch is an array built into the library; see include/dsa.h)."""
    return int(lib.dsa_sparse_mla_fwd_noalloc(
        ctypes.byref(pb.dims), ctypes.byref(pb.seqs), _ptr(q), _ptr(kv), _ptr(idx), row_begin,
        row_count, _ptr(out), _ptr(lse), _ptr(dev_status), _stream(stream)))


def dsa_forward_workspace_size(pb: Problem) -> int:
    return int(lib.dsa_forward_workspace_size(ctypes.byref(pb.dims), ctypes.byref(pb.seqs)))


def dsa_forward_workspace_size_for(pb: Problem, sm_count: int) -> int:
    return int(lib.dsa_forward_workspace_size_for(ctypes.byref(pb.dims), ctypes.byref(pb.seqs),
                                                  sm_count))


def dsa_forward_chunk_rows_for(pb: Problem, seq: int, sm_count: int) -> int:
    return int(lib.dsa_forward_chunk_rows_for(ctypes.byref(pb.dims), ctypes.byref(pb.seqs), seq,
                                              sm_count))


def dsa_forward(pb: Problem, q_idx, q_scale, w, k_idx, k_scale, q, kv, idx_out, out, lse,
                workspace, workspace_bytes: int, dev_status=None, stream=None,
                sel_out=None) -> int:
    return int(lib.dsa_forward(
        ctypes.byref(pb.dims), ctypes.byref(pb.seqs), _ptr(q_idx), _ptr(q_scale), _ptr(w),
        _ptr(k_idx), _ptr(k_scale), _ptr(q), _ptr(kv), _ptr(idx_out), _ptr(sel_out), _ptr(out),
        _ptr(lse), _ptr(workspace), workspace_bytes, _ptr(dev_status), _stream(stream)))


def dsa_forward_rows(pb: Problem, row_begin: int, row_count: int, q_idx, q_scale, w, k_idx,
                     k_scale, q, kv, idx_out, out, lse, workspace, workspace_bytes: int,
                     dev_status=None, stream=None, sel_out=None) -> int:
    return int(lib.dsa_forward_rows(
        ctypes.byref(pb.dims), ctypes.byref(pb.seqs), row_begin, row_count, _ptr(q_idx),
        _ptr(q_scale), _ptr(w), _ptr(k_idx), _ptr(k_scale), _ptr(q), _ptr(kv), _ptr(idx_out),
        _ptr(sel_out), _ptr(out), _ptr(lse), _ptr(workspace), workspace_bytes, _ptr(dev_status),
        _stream(stream)))


def dsa_cache_append(pb: Problem, k_new, kv_new, k_cache, k_scale_cache, kv_cache,
                     dev_status=None, stream=None) -> int:
    return int(lib.dsa_cache_append(
        ctypes.byref(pb.dims), ctypes.byref(pb.seqs), _ptr(k_new), _ptr(kv_new), _ptr(k_cache),
        _ptr(k_scale_cache), _ptr(kv_cache), _ptr(dev_status), _stream(stream)))


def dsa_indexer_kl_target(pb: Problem, q, kv, idx, lse, row_begin: int, row_count: int, target,
                          dev_status=None, stream=None) -> int:
    return int(lib.dsa_indexer_kl_target(
        ctypes.byref(pb.dims), ctypes.byref(pb.seqs), _ptr(q), _ptr(kv), _ptr(idx), _ptr(lse),
        row_begin, row_count, _ptr(target), _ptr(dev_status), _stream(stream)))


def dsa_indexer_kl_backward(pb: Problem, q_idx, q_scale, w, k_idx, k_scale, idx, target,
                            row_begin: int, row_count: int, loss, dw, dq, dk, dev_status=None,
                            stream=None, sel=None) -> int:
    """sel: optional [row_count, topk] scores of the selected keys (the forward's sel_out)."""
    return int(lib.dsa_indexer_kl_backward(
        ctypes.byref(pb.dims), ctypes.byref(pb.seqs), _ptr(q_idx), _ptr(q_scale), _ptr(w),
        _ptr(k_idx), _ptr(k_scale), _ptr(idx), _ptr(sel), _ptr(target), row_begin, row_count,
        _ptr(loss), _ptr(dw), _ptr(dq), _ptr(dk), _ptr(dev_status), _stream(stream)))


def dsa_indexer_kl_target_dense(pb: Problem, q, kv, lse, row_begin: int, row_count: int, target,
                                ld_target: int, dev_status=None, stream=None) -> int:
    return int(lib.dsa_indexer_kl_target_dense(
        ctypes.byref(pb.dims), ctypes.byref(pb.seqs), _ptr(q), _ptr(kv), _ptr(lse), row_begin,
        row_count, _ptr(target), ld_target, _ptr(dev_status), _stream(stream)))


def dsa_indexer_kl_backward_dense(pb: Problem, q_idx, q_scale, w, k_idx, k_scale, target,
                                  ld_target: int, row_begin: int, row_count: int, loss, dw, dq,
                                  dk, dev_status=None, stream=None) -> int:
    return int(lib.dsa_indexer_kl_backward_dense(
        ctypes.byref(pb.dims), ctypes.byref(pb.seqs), _ptr(q_idx), _ptr(q_scale), _ptr(w),
        _ptr(k_idx), _ptr(k_scale), _ptr(target), ld_target, row_begin, row_count, _ptr(loss),
        _ptr(dw), _ptr(dq), _ptr(dk), _ptr(dev_status), _stream(stream)))


def dsa_selftest_wait_timeout(dev_status, stream=None) -> int:
    return int(lib.dsa_selftest_wait_timeout(_ptr(dev_status), _stream(stream)))


def dsa_probe_dsmem(clusters: int, bytes_: int, reps: int, ns, bad, stream=None) -> int:
    return int(lib.dsa_probe_dsmem(clusters, bytes_, reps, _ptr(ns), _ptr(bad), _stream(stream)))


def dsa_probe_page_stream(k_blocks, block_ids, n_blocks: int, d_idx: int, ctas_per_sm: int,
                          bad, stream=None) -> int:
    return int(lib.dsa_probe_page_stream(_ptr(k_blocks), _ptr(block_ids), block_ids.numel(),
                                         n_blocks, d_idx, ctas_per_sm, _ptr(bad),
                                         _stream(stream)))


def dsa_read_device_status(dev_status, stream=None):
    raw = ctypes.c_int32(0)
    st = int(lib.dsa_read_device_status(_ptr(dev_status), _stream(stream), ctypes.byref(raw)))
    return st, int(raw.value)


# ---------------------------------------------------------------------- convenience

def check(status: int, what: str = "") -> None:
    if status != DSA_OK:
        raise DsaError(status, what)


class Forward:
    """Owns the outputs and workspace of ``dsa_forward`` for one workload shape (allocated with
    torch, once), so repeated calls allocate nothing."""

    def __init__(self, wl, keep_idx: bool = True, keep_sel: bool = False):
        dev = wl.q.device
        d = wl.dims
        T = wl.total_rows
        self.wl = wl
        self.pb = problem_of(wl)
        self.ws_bytes = dsa_forward_workspace_size(self.pb)
        if self.ws_bytes == 0:
            raise DsaError(DSA_ERR_INVALID_ARG, "dsa_forward_workspace_size")
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.out = torch.empty(T, d["h"], d["d_v"], dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(T, d["h"], dtype=torch.float32, device=dev)
        self.idx = (torch.empty(T, d["topk"], dtype=torch.int32, device=dev)
                    if keep_idx else None)
        # the selected keys' scores (the indexer's training step takes them)
        self.sel = (torch.empty(T, d["topk"], dtype=torch.float32, device=dev)
                    if keep_idx and keep_sel else None)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def __call__(self, stream=None) -> int:
        wl = self.wl
        return dsa_forward(self.pb, wl.q_idx, wl.q_scale, wl.w, wl.k_idx, wl.k_scale, wl.q,
                           wl.kv, self.idx, self.out, self.lse, self.ws, self.ws_bytes,
                           self.status, stream, sel_out=self.sel)
