/*
 * dsa.h -- C ABI of the B200 (sm_100a) DeepSeek Sparse Attention hot path.
 *
 * The path has three stages, in the order "FP8 index -> top-k selection -> sparse core
 * attention" ("DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek Sparse Attention
 * (DSA)", pipeline summary):
 *
 *   dsa_indexer_scores  lightning indexer: for query row t and every prior key s <= pos(t)
 *                       of its sequence,
 *                         S[t,s] = k_scale[s] * sum_j w[t,j] * q_scale[t,j]
 *                                    * ReLU( sum_i q_idx[t,j,i] * k_idx[s,i] )
 *                       with e4m3 q_idx / k_idx and fp32 accumulation (the indexer "scores
 *                       context tokens", same page, two-stage attention path; "Lightning
 *                       Indexer computes lightweight index scores", maplevalley page,
 *                       section 1; the weighted sum of ReLU(q.k) over indexer heads is the
 *                       formula this library implements)
 *   dsa_topk            per query row, the topk keys with the largest S; equal scores go to
 *                       the smaller key index; rows with fewer than topk prior keys keep
 *                       all of them (top-k=2048, same page, "Training signal"; "the Top-k
 *                       selector keeps only k key-value pairs per query", maplevalley page,
 *                       section 1)
 *   dsa_sparse_mla_fwd  MLA in MQA mode over the selected latent rows: every selected
 *                       576-d latent row is shared by all query heads (same page,
 *                       "Instantiation"); logits sigma * q.kv, softmax, output = weighted
 *                       sum of the first d_v latent dims, plus the natural-log LSE
 *   dsa_forward         the three stages back to back, for prefill (packed varlen causal
 *                       rows) and decode (one new token per sequence, paged or contiguous
 *                       caches)
 *
 * and, around the path: dsa_cache_append (the decode step that writes the new token's e4m3
 * indexer key and latent row into the caches), and dsa_indexer_kl_target with
 * dsa_indexer_kl_backward (the indexer's training step in the sparse stage), each documented
 * where it is declared below.
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller, row-major and contiguous.
 *     The library allocates nothing and keeps no state apart from a per-device attribute
 *     cache.  dims / seqs structs are HOST pointers, read during the call only.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Argument errors are returned synchronously, before anything is launched.
 *     A failed launch returns DSA_ERR_CUDA.
 *   - `dev_status` is an optional caller-owned DEVICE int32.  Kernels OR in
 *     DSA_DEVICE_TIMEOUT when a bounded wait gave up (the kernel then unwinds instead of
 *     hanging) and DSA_DEVICE_BAD_INDEX when an index or block-table entry points outside
 *     the caches (that entry is then skipped).  Clear it before the call; read it with
 *     dsa_read_device_status.  NULL disables the reporting (the kernels still unwind).
 *   - Alignment: every tensor pointer must be 16-byte aligned, ld_scores a multiple of 4;
 *     otherwise DSA_ERR_MISALIGNED.
 *   - Supported shapes: (h_idx, d_idx) in {(64,128), (4,32)}; (h, d_qk, d_v) in
 *     {(128,576,512), (16,160,128)}; topk a multiple of 64 in [64, 2048]; block_size 64.
 *     Decode needs (h_idx, d_idx) = (64,128).  Anything else: DSA_ERR_UNSUPPORTED_SHAPE.
 *
 * Geometry (dsa_seqs_t):
 *   PREFILL: total_rows packed query rows; row r of sequence b (cu[b] <= r < cu[b+1]) has
 *            position pos = r - cu[b] and sees keys 0..pos of its own sequence, which are
 *            the same packed rows of k_idx / k_scale / kv (physical row cu[b] + s).
 *   DECODE : one query row per sequence b (total_rows = batch) at position seq_lens[b]-1;
 *            it sees keys 0..seq_lens[b]-1.  Logical key s of sequence b is physical row
 *            block_table[b, s / block_size] * block_size + s % block_size, or, with
 *            block_table == NULL, b * max_seqlen + s.
 *   Key indices returned by dsa_topk and consumed by dsa_sparse_mla_fwd are LOGICAL
 *   positions within the sequence.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_ABI_VERSION 3

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

typedef struct CUstream_st* dsa_stream_t; /* cudaStream_t */

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,         /* null pointer, negative size, inconsistent geometry */
  DSA_ERR_UNSUPPORTED_SHAPE = 2,   /* dims outside the supported set */
  DSA_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes below the *_workspace_size answer */
  DSA_ERR_MISALIGNED = 4,          /* pointer not 16-byte aligned or ld not a multiple of 4 */
  DSA_ERR_BAD_INDEX = 5,           /* device status: an index left the caches */
  DSA_ERR_TIMEOUT = 6,             /* device status: a bounded wait gave up */
  DSA_ERR_CUDA = 7                 /* a CUDA runtime call or launch failed */
} dsa_status_t;

/* Bits of the device status word. */
#define DSA_DEVICE_TIMEOUT 1
#define DSA_DEVICE_BAD_INDEX 2

enum { DSA_PREFILL = 0, DSA_DECODE = 1 };

typedef struct {
  int32_t h_idx;        /* indexer heads */
  int32_t d_idx;        /* indexer head dim (e4m3 bytes per key row) */
  int32_t h;            /* query heads */
  int32_t d_qk;         /* latent + RoPE dims of q and of a latent KV row */
  int32_t d_v;          /* value dims = the first d_v dims of a latent KV row */
  int32_t topk;         /* keys kept per query row */
  int32_t block_size;   /* page size of the decode caches (64) */
  float softmax_scale;  /* sigma in the logits sigma * q.kv */
} dsa_dims_t;

typedef struct {
  int32_t mode;                  /* DSA_PREFILL or DSA_DECODE */
  int32_t batch;                 /* sequences */
  int32_t total_rows;            /* query rows: prefill cu_seqlens[batch]; decode batch */
  int32_t max_seqlen;            /* longest sequence; decode without block table: row stride */
  int64_t num_kv_rows;           /* physical rows of k_idx, k_scale and kv */
  const int32_t* cu_seqlens;     /* PREFILL: device [batch+1], cu[0] = 0, non-decreasing */
  const int32_t* cu_seqlens_host;/* PREFILL: host copy of cu_seqlens, used for planning */
  const int32_t* seq_lens;       /* DECODE : device [batch], each in [1, max_seqlen] */
  const int32_t* block_table;    /* DECODE : device [batch, max_blocks] or NULL */
  int32_t max_blocks;            /* DECODE : columns of block_table */
} dsa_seqs_t;

/* Stage 1.  Scores of query rows [row_begin, row_begin + row_count) against their prior
 * keys.  PREFILL rows may span several sequences.
 *   q_idx   e4m3 [total_rows, h_idx, d_idx]      q_scale, w  fp32 [total_rows, h_idx]
 *   k_idx   e4m3 [num_kv_rows, d_idx]            k_scale     fp32 [num_kv_rows]
 *   scores  fp32 [row_count, ld_scores]: scores[(t - row_begin) * ld + s] for s <= pos(t);
 *           entries past pos(t) are left untouched.  ld_scores >= max pos(t) + 1 over
 *           the rows and a multiple of 4.
 *   hist    optional uint32 [row_count, DSA_TOPK_HIST_BINS], zero on entry: the indexer ADDS
 *           to row t - row_begin the count of each written score in the bin of its first
 *           radix digit (the top 11 bits of the order-preserving key the selection sorts on),
 *           so that dsa_topk can start from exact per-row counts (the fused indexer + top-k).
 *           (64, 128) indexer only: with (4, 32) a non-NULL hist is DSA_ERR_UNSUPPORTED_SHAPE.
 *           NULL: no counting. */
#define DSA_TOPK_HIST_BINS 2048
DSA_API dsa_status_t dsa_indexer_scores(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                const uint8_t* q_idx, const float* q_scale, const float* w,
                                const uint8_t* k_idx, const float* k_scale, int32_t row_begin,
                                int32_t row_count, float* scores, int64_t ld_scores,
                                uint32_t* hist, int32_t* dev_status, dsa_stream_t stream);

/* Stage 2.  Exact top-k of each row of `scores` (layout as written by dsa_indexer_scores)
 * over keys 0..pos(t).  idx int32 [row_count, topk]: the selected LOGICAL key indices in
 * increasing order, then -1 padding when pos(t) + 1 < topk.  The set is unique: larger
 * score first, equal scores broken by the smaller index (-0 and +0 compare equal).
 *   hist  optional: the histograms dsa_indexer_scores counted while writing these same rows
 *         of `scores` (exact counts of each row's keys 0..pos(t); anything else gives a wrong
 *         selection).  The selection then starts from them and reads each score once; on
 *         return they are zero again, ready for the next dsa_indexer_scores.  NULL: the
 *         selection counts the first digit itself (one more read of the scores).
 *   sel_out  optional fp32 [row_count, topk]: the score of each selected key (sel_out[t][e] =
 *         scores[t][idx[t][e]], the value the selection compared), 0 where idx is -1; the
 *         indexer's training step takes them (dsa_indexer_kl_backward).  NULL: not written. */
DSA_API dsa_status_t dsa_topk(const dsa_dims_t* dims, const dsa_seqs_t* seqs, const float* scores,
                      int64_t ld_scores, uint32_t* hist, int32_t row_begin, int32_t row_count,
                      int32_t* idx, float* sel_out, int32_t* dev_status, dsa_stream_t stream);

/* Stages 1 and 2 fused: the indexer scores of rows [row_begin, row_begin + row_count) and their
 * top-k, without the scores leaving the call.  The pages' selector keeps k tokens per query
 * straight from the indexer's scores ("FP8 index -> top-k selection -> sparse core attention",
 * "DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek Sparse Attention (DSA)", pipeline
 * summary; "the Top-k selector keeps only k key-value pairs per query", maplevalley page,
 * section 1).  As it writes each score into a slab in `workspace`, the indexer counts it in
 * its row's histogram of the first radix digit (the top 11 bits of the order-preserving key);
 * the selection then starts from those counts and reads the slab once.  Inputs as for
 * dsa_indexer_scores; idx and the optional sel_out as written by dsa_topk (the same set,
 * increasing order, -1 padding).
 * workspace: at least dsa_indexer_topk_workspace_size(dims, seqs, row_count) bytes, 16-byte
 * aligned, caller-owned, contents on entry irrelevant (too small: DSA_ERR_WORKSPACE_TOO_SMALL).
 * With the (4, 32) indexer shape the selection builds its histograms itself. */
DSA_API size_t dsa_indexer_topk_workspace_size(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                               int32_t row_count);
DSA_API dsa_status_t dsa_indexer_topk(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                      const uint8_t* q_idx, const float* q_scale, const float* w,
                                      const uint8_t* k_idx, const float* k_scale,
                                      int32_t row_begin, int32_t row_count, int32_t* idx,
                                      float* sel_out, void* workspace, size_t workspace_bytes,
                                      int32_t* dev_status, dsa_stream_t stream);

/* Bytes of workspace dsa_sparse_mla_fwd needs for `row_count` rows (split-KV partials when
 * few rows leave SMs idle).  0 is a valid answer. */
DSA_API size_t dsa_sparse_mla_workspace_size(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                     int32_t row_count);

/* The same size for a device with `sm_count` SMs, without touching any device (host-only), when
 * the partials may take at most `max_bytes` (SIZE_MAX: no limit, the answer
 * dsa_sparse_mla_workspace_size gives on such a device).  The split count only changes speed:
 * under a cap the fastest split count that fits is chosen, and one split needs no partials, so
 * the answer never exceeds max_bytes.  dsa_sparse_mla_fwd_noalloc sizes its partials this way
 * with max_bytes = DSA_NOALLOC_SCRATCH_BYTES.  0 on invalid arguments or sm_count <= 0. */
DSA_API size_t dsa_sparse_mla_workspace_size_for(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                                 int32_t row_count, int32_t sm_count,
                                                 size_t max_bytes);

/* Stage 3.  Sparse MLA-MQA forward for rows [row_begin, row_begin + row_count).
 *   q    bf16 [total_rows, h, d_qk]   (indexed by absolute row)
 *   kv   bf16 [num_kv_rows, d_qk]
 *   idx  int32 [row_count, topk] logical key indices (-1 = unused), relative to row_begin,
 *        or NULL: every prior key of each row (dense causal attention), which is exactly the
 *        top-k's selection when no row has more than topk prior keys, and the dense model's
 *        attention (the training's warm-up stage) when rows are longer.  PREFILL rows of any
 *        length; DECODE with NULL needs max_seqlen <= topk (else DSA_ERR_INVALID_ARG)
 *   out  bf16 [total_rows, h, d_v] and lse fp32 [total_rows, h] (absolute rows); a row
 *        with no valid index gets out = 0 and lse = -inf. */
DSA_API dsa_status_t dsa_sparse_mla_fwd(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                                int32_t row_begin, int32_t row_count, uint16_t* out,
                                float* lse, void* workspace, size_t workspace_bytes,
                                int32_t* dev_status, dsa_stream_t stream);

/* Sparse MLA forward for callers that cannot allocate device memory.  No counterpart on the
 * pages: it is a packaging of dsa_sparse_mla_fwd, not a step of the method.
 *
 * Some callers may not call cudaMalloc or any allocator at all: code recorded into a CUDA graph,
 * where an allocation would break the capture; runtimes that hand out every byte of device memory
 * from their own fixed pool; plugins whose host framework forbids allocator calls on the hot
 * path.  This entry point computes exactly what dsa_sparse_mla_fwd computes (same arguments
 * minus the workspace) and keeps its split-KV partials in a scratch array built into the
 * library: DSA_NOALLOC_SCRATCH_BYTES (20 MiB) of device memory that every GPU loading the
 * library holds until the process exits.
 *   - The first call on a device looks up that device's copy of the array
 *     (cudaGetSymbolAddress, with that device current).  Make that first call before any stream
 *     capture.
 *   - The split-KV slicing is chosen so that the partials fit the array: the fastest split
 *     count with splits * row_count * h * (d_v + 1) * 4 bytes (+256) within
 *     DSA_NOALLOC_SCRATCH_BYTES (at full shapes, splits * row_count <= 79), else one split,
 *     which needs no scratch at all.  Every row count therefore runs; large batches run
 *     unsplit, exactly as dsa_sparse_mla_fwd runs them.
 *   - Every call shares the one array and each call overwrites the parts it uses, so nothing has
 *     to start at zero; two calls that overlap on the GPU (different streams, no ordering) race
 *     on it and give undefined results.  Calls on one stream are safe. */
#define DSA_NOALLOC_SCRATCH_BYTES (20u << 20)
DSA_API dsa_status_t dsa_sparse_mla_fwd_noalloc(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                                const uint16_t* q, const uint16_t* kv,
                                                const int32_t* idx, int32_t row_begin,
                                                int32_t row_count, uint16_t* out, float* lse,
                                                int32_t* dev_status, dsa_stream_t stream);

/* Bytes of workspace dsa_forward needs (score slab for one row chunk, chunk indices when
 * idx_out is NULL, split-KV partials).  Larger workspaces allow larger prefill chunks. */
DSA_API size_t dsa_forward_workspace_size(const dsa_dims_t* dims, const dsa_seqs_t* seqs);

/* The same size for a device with `sm_count` SMs, without touching any device (host-only; for
 * sizing buffers before a device is chosen).  0 on invalid arguments or sm_count <= 0. */
DSA_API size_t dsa_forward_workspace_size_for(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                              int32_t sm_count);

/* How dsa_forward cuts a prefill into row chunks, for a device with `sm_count` SMs (host-only):
 * the rows per chunk of sequence `seq` (the last chunk of a sequence may be shorter; with
 * idx_out NULL the first min(L, topk) rows run dense attention before the chunks start).  Each
 * chunk is one indexer, one top-k and one attention launch over its rows.  DECODE: the batch
 * (one chunk).  0 on invalid arguments. */
DSA_API int32_t dsa_forward_chunk_rows_for(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                           int32_t seq, int32_t sm_count);

/* The whole path for all seqs->total_rows query rows.  Inputs as for the three stages.
 *   idx_out  optional int32 [total_rows, topk]: the selected indices (NULL = not kept).
 *            When NULL, rows with at most topk prior keys (the first topk rows of each prefill
 *            sequence; a decode batch whose max_seqlen <= topk) skip the indexer and the top-k,
 *            whose selection would be all of their keys, and run dense attention.
 *   sel_out  optional fp32 [total_rows, topk]: the indexer score of each selected key, as
 *            dsa_topk writes it (requires idx_out; else DSA_ERR_INVALID_ARG).
 *   out, lse as for dsa_sparse_mla_fwd. */
DSA_API dsa_status_t dsa_forward(const dsa_dims_t* dims, const dsa_seqs_t* seqs, const uint8_t* q_idx,
                         const float* q_scale, const float* w, const uint8_t* k_idx,
                         const float* k_scale, const uint16_t* q, const uint16_t* kv,
                         int32_t* idx_out, float* sel_out, uint16_t* out, float* lse,
                         void* workspace, size_t workspace_bytes, int32_t* dev_status,
                         dsa_stream_t stream);

/* dsa_forward for query rows [row_begin, row_begin + row_count) only, with the query-side
 * arrays holding just those rows: the building block of a prefill split across GPUs (each GPU
 * takes a range of query rows; the keys are gathered first, since every row attends to the
 * prior keys of its whole sequence).  The rows, chunks, selection and results are exactly those
 * dsa_forward computes for the same rows.
 *   q_idx [row_count, h_idx, d_idx], q_scale / w [row_count, h_idx], q [row_count, h, d_qk],
 *   out [row_count, h, d_v], lse [row_count, h], idx_out and sel_out (optional) [row_count,
 *   topk]: row i of these is query row row_begin + i.
 *   k_idx, k_scale, kv: the full key-side arrays (num_kv_rows physical rows), as for dsa_forward.
 *   workspace: dsa_forward_workspace_size(dims, seqs) bytes suffice for every row range.
 * DECODE: rows are sequences (a range of the batch). */
DSA_API dsa_status_t dsa_forward_rows(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                      int32_t row_begin, int32_t row_count,
                                      const uint8_t* q_idx, const float* q_scale, const float* w,
                                      const uint8_t* k_idx, const float* k_scale,
                                      const uint16_t* q, const uint16_t* kv, int32_t* idx_out,
                                      float* sel_out, uint16_t* out, float* lse, void* workspace,
                                      size_t workspace_bytes, int32_t* dev_status,
                                      dsa_stream_t stream);

/* Decode cache append, the step that fills the caches the path reads ("FP8 index -> top-k
 * selection -> sparse core attention", "DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek
 * Sparse Attention (DSA)", pipeline summary: the indexer reads keys in FP8).  DECODE mode only.
 * For each sequence b the new token sits at position p = seq_lens[b] - 1 (the lengths already
 * count it); it is written at physical row block_table[b][p / block_size] * block_size +
 * p % block_size, or b * max_seqlen + p when block_table is NULL:
 *   k_new     fp32 [batch, d_idx]: the new token's indexer key, quantised per token: scale =
 *             amax / 448 in fp32 (1 when amax = 0), codes = the e4m3 value nearest to x / scale
 *             (ties to even, saturating at +-448)
 *   kv_new    bf16 [batch, d_qk]: the new token's latent row, copied unchanged
 *   k_cache   e4m3 [num_kv_rows, d_idx], k_scale_cache fp32 [num_kv_rows], kv_cache bf16
 *             [num_kv_rows, d_qk]: caller-owned caches, written at the one row per sequence
 * All pointers 16-byte aligned.  An entry whose position or block falls outside the caches is
 * skipped and sets DSA_DEVICE_BAD_INDEX in *dev_status. */
DSA_API dsa_status_t dsa_cache_append(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                      const float* k_new, const uint16_t* kv_new,
                                      uint8_t* k_cache, float* k_scale_cache, uint16_t* kv_cache,
                                      int32_t* dev_status, dsa_stream_t stream);

/* ---- indexer training (sparse stage) ------------------------------------------------------
 * The indexer is trained to imitate the main attention's head-summed distribution through a KL
 * divergence ("DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek Sparse Attention (DSA)",
 * "Training signal"); in the sparse stage both distributions live on each row's selected keys.
 * Two calls give one training step of the indexer after a forward pass that kept its indices
 * and LSE: the target, then the loss with the gradients. */

/* Target of rows [row_begin, row_begin + row_count):
 *   target[t - row_begin, e] = (1/h) sum_h exp(sigma q[t,h,:] . kv[idx[t,e], :] - lse[t,h])
 * (each head's attention distribution over the selection, averaged over heads; with the LSE
 * of the forward pass over the same selection every row sums to 1).
 *   q, kv, idx   as for dsa_sparse_mla_fwd (idx relative to row_begin; NULL = every prior key,
 *                allowed only when no row has more than topk prior keys)
 *   lse          fp32 [total_rows, h]: the forward's LSE (natural log, sigma applied)
 *   target       fp32 [row_count, topk], caller-owned; entries with idx = -1 are set to 0
 * Shapes as for dsa_sparse_mla_fwd.  All pointers 16-byte aligned.  Out-of-range indices are
 * skipped (target 0) and set DSA_DEVICE_BAD_INDEX; timeouts set DSA_DEVICE_TIMEOUT. */
DSA_API dsa_status_t dsa_indexer_kl_target(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                           const uint16_t* q, const uint16_t* kv,
                                           const int32_t* idx, const float* lse,
                                           int32_t row_begin, int32_t row_count, float* target,
                                           int32_t* dev_status, dsa_stream_t stream);

/* KL loss of the indexer against `target` on the selected keys, and its gradients.  With the
 * real-valued inputs q = q_scale * q_idx (per row and head) and k = k_scale * k_idx (per key),
 * per row t over the entries e with idx[t,e] >= 0:
 *   D[j,e] = q[t,j,:] . k[idx[t,e],:],  S_e = sum_j w[t,j] max(D[j,e], 0)  (the indexer score)
 *   pi = softmax(S),  loss[t] = sum_e p_e (ln p_e - ln pi_e)  (p = target row, 0 ln 0 = 0)
 *   g_e = pi_e sum_f p_f - p_e
 *   dw[t,j]    = sum_e g_e max(D[j,e], 0)
 *   dq[t,j,:]  = w[t,j] sum_e g_e [D[j,e] > 0] k[idx[t,e],:]
 *   dk[row,:] += g_e sum_j w[t,j] [D[j,e] > 0] q[t,j,:]   for the physical row of idx[t,e]
 * (d/dx max(x, 0) = 0 at x = 0; the gradients are those of the real values, so a caller that
 * quantised q and k passes them straight through the rounding).
 *   q_idx, q_scale, w, k_idx, k_scale   as for dsa_indexer_scores (k_scale must not be NULL;
 *            the scales must be positive, as the e4m3 quantiser makes them: the ReLU masks
 *            are taken from the e4m3 products)
 *   idx      int32 [row_count, topk], relative to row_begin, -1 = unused (required)
 *   sel_scores  optional fp32 [row_count, topk]: the indexer scores S of the selected keys, as
 *            the forward's selection wrote them (dsa_topk, dsa_indexer_topk, dsa_forward
 *            sel_out).  Given, pi is the softmax of these values and the keys are read once
 *            (the D products are still recomputed for the ReLU masks and the gradients); NULL:
 *            S is recomputed from q and k (two reads of the keys).  Both agree up to rounding.
 *   target   fp32 [row_count, topk]
 *   loss     fp32 [row_count];  dw fp32 [row_count, h_idx];  dq fp32 [row_count, h_idx, d_idx]
 *   dk       fp32 [num_kv_rows, d_idx]: ADDED to (zero it first); the order of the atomic
 *            additions is not fixed, so its last bits may vary from run to run
 * Indexer shapes (h_idx, d_idx) = (64, 128) with topk a multiple of 128, or (4, 32); both
 * modes.  All pointers 16-byte aligned.  Out-of-range indices are skipped and set
 * DSA_DEVICE_BAD_INDEX. */
DSA_API dsa_status_t dsa_indexer_kl_backward(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                             const uint8_t* q_idx, const float* q_scale,
                                             const float* w, const uint8_t* k_idx,
                                             const float* k_scale, const int32_t* idx,
                                             const float* sel_scores, const float* target,
                                             int32_t row_begin, int32_t row_count, float* loss,
                                             float* dw, float* dq, float* dk,
                                             int32_t* dev_status, dsa_stream_t stream);

/* The dense warm-up stage of the indexer's training ("DeepSeek V3.2-Exp Cuts Long-Context Costs
 * with DeepSeek Sparse Attention (DSA)", "Training signal": before the sparse stage the indexer
 * learns to imitate the dense attention, over every prior key).  PREFILL only.  The entries of
 * query row t are its keys 0..pos(t), in position order; target rows have one entry per key.
 *
 * Target: target[t - row_begin, s] = (1/h) sum_h exp(sigma q[t,h,:] . kv[s,:] - lse[t,h]) for
 * s <= pos(t), with lse from dsa_sparse_mla_fwd with idx = NULL (the dense attention of the
 * same rows).  target fp32 [row_count, ld_target], ld_target a multiple of 64 (else
 * DSA_ERR_MISALIGNED), at least topk and the longest row's key count rounded up to 64 (else
 * DSA_ERR_INVALID_ARG); entries past pos(t) are 0 or left untouched. */
DSA_API dsa_status_t dsa_indexer_kl_target_dense(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                                 const uint16_t* q, const uint16_t* kv,
                                                 const float* lse, int32_t row_begin,
                                                 int32_t row_count, float* target,
                                                 int64_t ld_target, int32_t* dev_status,
                                                 dsa_stream_t stream);

/* Loss and gradients of the same KL as dsa_indexer_kl_backward, over every prior key of each row
 * (entry s = key s, target [row_count, ld_target] as written by dsa_indexer_kl_target_dense,
 * ld_target a multiple of 4 and at least the longest row's key count).  Outputs as for
 * dsa_indexer_kl_backward.  The (64, 128) indexer takes rows of any length; the (4, 32) shape
 * rows of at most 2048 keys (else DSA_ERR_UNSUPPORTED_SHAPE). */
DSA_API dsa_status_t dsa_indexer_kl_backward_dense(const dsa_dims_t* dims,
                                                   const dsa_seqs_t* seqs, const uint8_t* q_idx,
                                                   const float* q_scale, const float* w,
                                                   const uint8_t* k_idx, const float* k_scale,
                                                   const float* target, int64_t ld_target,
                                                   int32_t row_begin, int32_t row_count,
                                                   float* loss, float* dw, float* dq, float* dk,
                                                   int32_t* dev_status, dsa_stream_t stream);

/* Synchronises `stream`, reads the device status word and maps it: 0 -> DSA_OK,
 * DSA_DEVICE_TIMEOUT -> DSA_ERR_TIMEOUT, DSA_DEVICE_BAD_INDEX -> DSA_ERR_BAD_INDEX.
 * *raw (optional, host) receives the word. */
DSA_API dsa_status_t dsa_read_device_status(const int32_t* dev_status, dsa_stream_t stream,
                                    int32_t* raw);

/* Diagnostics: checks that a wait which never completes ends instead of hanging.  Launches one
 * CTA of two warps that wait, with the same bounded wait every kernel above uses (2 s limit), on
 * an mbarrier nothing arrives at; each warp that gives up ORs DSA_DEVICE_TIMEOUT into
 * *dev_status (device, 4-byte aligned, caller-owned) and the CTA then exits normally, leaving the
 * context usable.  Asynchronous on `stream`, which stays busy for about 2 s; read the word with
 * dsa_read_device_status, which then returns DSA_ERR_TIMEOUT. */
DSA_API dsa_status_t dsa_selftest_wait_timeout(int32_t* dev_status, dsa_stream_t stream);

/* Diagnostics: the rate of distributed-shared-memory traffic between the two CTAs of a cluster,
 * the figure that decides whether the two CTAs of an attention row can exchange partial logits
 * instead of each computing all of them.  Launches `clusters` clusters of two 512-thread CTAs
 * (one CTA per SM); the two CTAs of each cluster store `bytes` (a multiple of 16, at most the
 * device's shared memory per CTA) of 16-byte words into each other's shared memory `reps` times,
 * both at once.  ns (device, uint64 [clusters]) receives each cluster's exchange time in
 * nanoseconds; bad (device int32, zero it first) receives the count of words that did not land
 * as written (0 expected).  Asynchronous on `stream`. */
DSA_API dsa_status_t dsa_probe_dsmem(int32_t clusters, int32_t bytes, int32_t reps, uint64_t* ns,
                                     int32_t* bad, dsa_stream_t stream);

/* Diagnostics: the read rate of the decode indexer's key stream with no arithmetic, the
 * practical ceiling of that access pattern.  Reads pages of an interleaved indexer key cache
 * (k_blocks, device, 16-byte aligned, n_blocks pages of 64 key rows of d_idx bytes followed by
 * their 64 fp32 scales; d_idx 32 or 128) in the order of block_ids (device int32 [n_ids]: page
 * ids, e.g. the block-table rows of a decode batch) into shared memory with the indexer
 * producer's copies (one TMA box for the rows, one bulk copy for the scales) and discards them.
 * ctas_per_sm (1..8) CTAs per SM, each taking a contiguous range of block_ids and keeping as many
 * pages in flight as fit its share of the SM's shared memory (at most 32;
 * DSA_ERR_UNSUPPORTED_SHAPE when fewer than 2 fit).  An id outside [0, n_blocks) is skipped; bad
 * (device int32, zero it first) receives the number of skipped ids plus one per CTA whose bounded
 * wait ran out (0 expected).  Nothing is written but *bad.  Asynchronous on `stream`: time it
 * with events on that stream. */
DSA_API dsa_status_t dsa_probe_page_stream(const void* k_blocks, const int32_t* block_ids,
                                           int64_t n_ids, int64_t n_blocks, int32_t d_idx,
                                           int32_t ctas_per_sm, int32_t* bad,
                                           dsa_stream_t stream);

DSA_API const char* dsa_status_string(dsa_status_t status);

/* DSA_ABI_VERSION of the built library.  2: first-digit histograms (hist of dsa_indexer_scores
 * and dsa_topk), dsa_indexer_topk, dsa_forward_rows, the dense warm-up entry points;
 * 3: the scores of the selected keys (sel_out of dsa_topk, dsa_indexer_topk, dsa_forward and
 * dsa_forward_rows; sel_scores of dsa_indexer_kl_backward). */
DSA_API int32_t dsa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
