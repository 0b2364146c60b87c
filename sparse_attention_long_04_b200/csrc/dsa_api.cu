// C ABI of the DSA hot path (see include/dsa.h): argument checks, planning and launches.
// Nothing here allocates device memory; the only state is a per-device attribute cache.
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <climits>
#include <cstring>
#include <mutex>

#include "dsa.h"
#include "cache_append.cuh"
#include "indexer.cuh"
#include "indexer_bwd.cuh"
#include "indexer_bwd_tc.cuh"
#include "sparse_mla.cuh"
#include "topk.cuh"

namespace {

using namespace dsa;

constexpr int kMaxDevices = 64;
constexpr size_t kSlabBudget = size_t(256) << 20;  // prefill score slab per row chunk

struct DeviceInfo {
  int sm_count = 0;
  int max_smem = 0;
};

std::mutex g_mu;
DeviceInfo g_info[kMaxDevices];
bool g_info_ok[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

dsa_status_t device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_info_ok[dev]) {
    DeviceInfo d;
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
      return DSA_ERR_CUDA;
    g_info[dev] = d;
    g_info_ok[dev] = true;
  }
  *out = g_info[dev];
  return DSA_OK;
}

dsa_status_t encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode == nullptr) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr)
      return DSA_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  *fn = g_encode;
  return DSA_OK;
}

// Per (kernel, device): the dynamic shared-memory limit the kernel has been raised to.
struct SmemRaised {
  const void* fn;
  int bytes[kMaxDevices];
};
SmemRaised g_raised[32];
int g_n_raised = 0;

// Raises the kernel's dynamic shared-memory limit to at least smem_bytes on the current device
// (once per size increase).
template <typename Kernel>
dsa_status_t prepare_kernel(Kernel k, int smem_bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  const void* fn = reinterpret_cast<const void*>(k);
  std::lock_guard<std::mutex> lk(g_mu);
  int slot = -1;
  for (int i = 0; i < g_n_raised; ++i)
    if (g_raised[i].fn == fn) slot = i;
  if (slot >= 0 && g_raised[slot].bytes[dev] >= smem_bytes) return DSA_OK;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  if (slot < 0) {
    if (g_n_raised == 32) return DSA_OK;   // not cached: raised again next time
    slot = g_n_raised++;
    g_raised[slot] = SmemRaised{fn, {}};
  }
  g_raised[slot].bytes[dev] = smem_bytes;
  return DSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// NVTX range around an entry point (host side: argument checks, planning and the launches it
// enqueues); a no-op unless a profiler is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Launch with programmatic stream serialization: the kernel may start while the previous kernel
// of the stream is finishing; it waits for it (griddepcontrol.wait) before reading anything.
template <typename Kernel, typename... Args>
dsa_status_t launch_pdl(Kernel k, dim3 grid, int threads, int smem, cudaStream_t st,
                        Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k, args...) != cudaSuccess) return DSA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status_t launch_status() {
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ------------------------------------------------------------------------ argument checks

bool indexer_shape_ok(const dsa_dims_t& d, int mode) {
  if (d.h_idx == 64 && d.d_idx == 128) return true;
  return mode == DSA_PREFILL && d.h_idx == 4 && d.d_idx == 32;
}

bool mla_shape_ok(const dsa_dims_t& d) {
  return (d.h == 128 && d.d_qk == 576 && d.d_v == 512) ||
         (d.h == 16 && d.d_qk == 160 && d.d_v == 128);
}

dsa_status_t check_common(const dsa_dims_t* dims, const dsa_seqs_t* seqs) {
  if (dims == nullptr || seqs == nullptr) return DSA_ERR_INVALID_ARG;
  const dsa_seqs_t& s = *seqs;
  if (s.mode != DSA_PREFILL && s.mode != DSA_DECODE) return DSA_ERR_INVALID_ARG;
  if (s.batch <= 0 || s.total_rows < 0 || s.max_seqlen <= 0 || s.num_kv_rows <= 0)
    return DSA_ERR_INVALID_ARG;
  if (dims->topk < 64 || dims->topk > 2048 || dims->topk % 64 != 0)
    return DSA_ERR_UNSUPPORTED_SHAPE;
  if (s.mode == DSA_PREFILL) {
    if (s.cu_seqlens == nullptr || s.cu_seqlens_host == nullptr) return DSA_ERR_INVALID_ARG;
    const int32_t* cu = s.cu_seqlens_host;
    if (cu[0] != 0 || cu[s.batch] != s.total_rows) return DSA_ERR_INVALID_ARG;
    for (int b = 0; b < s.batch; ++b) {
      const int L = cu[b + 1] - cu[b];
      if (L < 0 || L > s.max_seqlen) return DSA_ERR_INVALID_ARG;
    }
    if (s.total_rows > s.num_kv_rows) return DSA_ERR_INVALID_ARG;
  } else {
    if (s.seq_lens == nullptr || s.total_rows != s.batch) return DSA_ERR_INVALID_ARG;
    if (dims->block_size != 64) return DSA_ERR_UNSUPPORTED_SHAPE;
    if (s.block_table != nullptr) {
      if (s.max_blocks < ceil_div(s.max_seqlen, 64)) return DSA_ERR_INVALID_ARG;
    } else if (static_cast<int64_t>(s.batch) * s.max_seqlen > s.num_kv_rows) {
      return DSA_ERR_INVALID_ARG;
    }
  }
  return DSA_OK;
}

dsa_status_t check_rows(const dsa_seqs_t* s, int32_t row_begin, int32_t row_count) {
  if (row_begin < 0 || row_count < 0 || row_begin + int64_t(row_count) > s->total_rows)
    return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

// Largest key count (pos + 1) among rows [row_begin, row_begin + row_count).
int64_t max_keys(const dsa_seqs_t* s, int32_t row_begin, int32_t row_count) {
  if (s->mode == DSA_DECODE) return s->max_seqlen;
  const int32_t* cu = s->cu_seqlens_host;
  int64_t m = 0;
  for (int b = 0; b < s->batch; ++b) {
    const int64_t lo = std::max<int64_t>(cu[b], row_begin);
    const int64_t hi = std::min<int64_t>(cu[b + 1], int64_t(row_begin) + row_count);
    if (lo < hi) m = std::max<int64_t>(m, hi - cu[b]);
  }
  return m;
}

// Without an index array attention runs dense: every prior key of each row (the top-k's
// selection when no row has more than topk prior keys; dense causal attention in general).
// Decode rows take at most topk keys that way (resolved through the block table up front);
// prefill rows of any length (their keys are consecutive packed rows, streamed past topk).
bool dense_ok(const dsa_dims_t& d, const dsa_seqs_t* s, int32_t row_begin, int32_t row_count) {
  return s->mode == DSA_PREFILL || max_keys(s, row_begin, row_count) <= d.topk;
}

// The training target without indices writes topk entries per row: rows of at most topk keys.
bool dense_target_ok(const dsa_dims_t& d, const dsa_seqs_t* s, int32_t row_begin,
                     int32_t row_count) {
  return max_keys(s, row_begin, row_count) <= d.topk;
}

// ------------------------------------------------------------------------ TMA maps

dsa_status_t make_map(CUtensorMap* map, const void* base, uint64_t rows, uint32_t row_bytes,
                      uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  if (encoder(&enc) != DSA_OK) return DSA_ERR_CUDA;
  std::memset(map, 0, sizeof(*map));
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {row_bytes, box_rows};
  cuuint32_t es[2] = {1, 1};
  const CUtensorMapSwizzle sw =
      row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                   strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DSA_OK : DSA_ERR_CUDA;
}

// Interleaved paged indexer cache: blocks of 64 key rows (row_bytes each) followed by their 64
// fp32 scales; one box = one block's 64 key rows.
dsa_status_t make_block_map(CUtensorMap* map, const void* base, uint64_t blocks,
                            uint32_t row_bytes) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  if (encoder(&enc) != DSA_OK) return DSA_ERR_CUDA;
  std::memset(map, 0, sizeof(*map));
  cuuint64_t dims[3] = {row_bytes, 64, blocks};
  cuuint64_t strides[2] = {row_bytes, uint64_t(64) * (row_bytes + 4)};
  cuuint32_t box[3] = {row_bytes, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw =
      row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                   strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DSA_OK : DSA_ERR_CUDA;
}

// The indexer's scales may live inside the key blocks (k_scale NULL) only in paged decode.
bool interleaved_ok(const dsa_seqs_t& s) {
  return s.mode == DSA_DECODE && s.block_table != nullptr && s.num_kv_rows % 64 == 0;
}

// Rows of `row_bytes` bytes (a multiple of 16), boxes of box_bytes x box_rows, 128-byte swizzle.
dsa_status_t make_row_map(CUtensorMap* map, const void* base, uint64_t rows, uint32_t row_bytes,
                          uint32_t box_bytes, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  if (encoder(&enc) != DSA_OK) return DSA_ERR_CUDA;
  std::memset(map, 0, sizeof(*map));
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_bytes, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                   strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DSA_OK : DSA_ERR_CUDA;
}

// ------------------------------------------------------------------------ stage 1

template <int H_I, int D_I, int QPG>
dsa_status_t run_indexer_kernel(const CUtensorMap& kmap, const CUtensorMap& qmap,
                                const IndexerParams& prm, dim3 grid, cudaStream_t st) {
  using C = IndexerCfg<H_I, D_I, QPG>;
  int smem = C::SMEM_BYTES;
  if (C::TMEM_COLS == 512) smem = std::max(smem, 120 * 1024);   // one CTA per SM
  auto k = dsa_indexer_kernel<H_I, D_I, QPG>;
  if (prepare_kernel(k, smem) != DSA_OK) return DSA_ERR_CUDA;
  // may launch while the previous kernel finishes (the kernel waits for it before any read)
  return launch_pdl(k, grid, C::THREADS, smem, st, kmap, qmap, prm);
}

// Key tiles per CTA of the decode indexer.  The launch is HBM-bound and every CTA streams
// tps tiles, so its time is about waves x (tps + c0): waves = ceil(rows x splits / slots) for
// `slots` resident CTAs, c0 ~ 2 tiles of per-CTA set-up (barriers, TMEM, the query group).
// Pick the split count with the smallest such makespan, so that the last wave is not a thin
// tail of a few CTAs.
int64_t decode_tiles_per_split(int64_t rows, int64_t tiles, int64_t slots) {
  int64_t best_tps = tiles;
  double best = 1e300;
  for (int64_t sp = 1; sp <= tiles; ++sp) {
    const int64_t tps = ceil_div(tiles, sp);
    if (sp > 1 && tps == ceil_div(tiles, sp - 1)) continue;   // same split as sp - 1
    const double waves = double(ceil_div(rows * ceil_div(tiles, tps), std::max<int64_t>(1, slots)));
    const double t = waves * (double(tps) + 2.0);
    if (t < best - 1e-9) {
      best = t;
      best_tps = tps;
    }
  }
  return best_tps;
}

template <int H_I, int D_I, int QPG>
dsa_status_t indexer_impl(const dsa_dims_t& d, const dsa_seqs_t& s, const uint8_t* q_idx,
                          const float* q_scale, const float* w, const uint8_t* k_idx,
                          const float* k_scale, int32_t row_begin, int32_t row_count,
                          float* scores, int64_t ld, int32_t* status, cudaStream_t st,
                          uint32_t* hist) {
  using C = IndexerCfg<H_I, D_I, QPG>;
  DeviceInfo info;
  if (device_info(&info) != DSA_OK) return DSA_ERR_CUDA;
  CUtensorMap kmap, qmap;
  // prefill keys are contiguous: one 128-row box per tile; decode: 64-row (paged) boxes; with
  // the scales inside the blocks, one 3-D box per block
  if (k_scale == nullptr) {
    if (make_block_map(&kmap, k_idx, uint64_t(s.num_kv_rows / 64), D_I) != DSA_OK)
      return DSA_ERR_CUDA;
  } else if (make_map(&kmap, k_idx, s.num_kv_rows, D_I, s.mode == DSA_DECODE ? 64 : 128) !=
             DSA_OK) {
    return DSA_ERR_CUDA;
  }
  if (make_map(&qmap, q_idx, uint64_t(s.total_rows) * H_I, D_I, C::N) != DSA_OK)
    return DSA_ERR_CUDA;
  IndexerParams prm{};
  prm.q_scale = q_scale;
  prm.w = w;
  prm.k_scale = k_scale;
  prm.k_blocks = k_idx;
  prm.scores = scores;
  prm.ld = ld;
  prm.status = status;
  prm.seq_lens = s.seq_lens;
  prm.block_table = s.block_table;
  prm.max_blocks = s.max_blocks;
  prm.kv_stride = s.max_seqlen;
  prm.max_seqlen = s.max_seqlen;
  prm.num_kv_rows = s.num_kv_rows;
  prm.hist = C::HIST ? hist : nullptr;
  const int ctas_per_sm = C::TMEM_COLS == 512 ? 1 : 2;
  const int64_t target = int64_t(info.sm_count) * ctas_per_sm * 4;
  if (s.mode == DSA_DECODE) {
    const int64_t tiles = ceil_div(s.max_seqlen, 128);
    const int64_t tps = decode_tiles_per_split(row_count, tiles, int64_t(info.sm_count) * ctas_per_sm);
    const int64_t splits = ceil_div(tiles, tps);
    prm.decode = 1;
    prm.row0 = row_begin;
    prm.nrows = row_count;
    prm.out_row0 = 0;
    prm.tiles_per_split = static_cast<int32_t>(tps);
    return run_indexer_kernel<H_I, D_I, QPG>(kmap, qmap, prm, dim3(row_count, splits), st);
  }
  // prefill: one launch per sequence segment of the row range
  const int32_t* cu = s.cu_seqlens_host;
  for (int b = 0; b < s.batch; ++b) {
    const int64_t lo = std::max<int64_t>(cu[b], row_begin);
    const int64_t hi = std::min<int64_t>(cu[b + 1], int64_t(row_begin) + row_count);
    if (lo >= hi) continue;
    const int64_t nrows = hi - lo;
    const int64_t groups = ceil_div(nrows, QPG);
    const int64_t tiles = ceil_div(hi - cu[b], 128);
    int64_t splits = std::min<int64_t>(tiles, std::max<int64_t>(1, ceil_div(target, groups)));
    const int64_t tps = std::max<int64_t>(ceil_div(tiles, splits), std::min<int64_t>(tiles, 8));
    splits = ceil_div(tiles, tps);
    prm.decode = 0;
    prm.row0 = static_cast<int32_t>(lo);
    prm.nrows = static_cast<int32_t>(nrows);
    prm.pos0 = static_cast<int32_t>(lo - cu[b]);
    prm.key0 = cu[b];
    prm.out_row0 = static_cast<int32_t>(lo - row_begin);
    prm.tiles_per_split = static_cast<int32_t>(tps);
    dsa_status_t e = run_indexer_kernel<H_I, D_I, QPG>(kmap, qmap, prm, dim3(groups, splits), st);
    if (e != DSA_OK) return e;
  }
  return DSA_OK;
}

dsa_status_t topk_launch(const dsa_dims_t& d, const dsa_seqs_t& s, const float* scores, int64_t ld,
                         int32_t row_begin, int32_t row_count, int32_t* idx, int32_t* status,
                         cudaStream_t st, uint32_t* hist = nullptr, float* sel = nullptr);

// Whether the indexer of these dims counts the first-digit histograms (the full 64 x 128 shape;
// the 4 x 32 shape's 64-row query groups have no room for them).
bool indexer_counts_hist(const dsa_dims_t& d) { return d.h_idx == 64 && d.d_idx == 128; }

dsa_status_t indexer_dispatch(const dsa_dims_t& d, const dsa_seqs_t& s, const uint8_t* q_idx,
                              const float* q_scale, const float* w, const uint8_t* k_idx,
                              const float* k_scale, int32_t row_begin, int32_t row_count,
                              float* scores, int64_t ld, int32_t* status, cudaStream_t st,
                              uint32_t* hist = nullptr) {
  if (row_count == 0) return DSA_OK;
  if (d.h_idx == 64 && d.d_idx == 128) {
    if (s.mode == DSA_DECODE)
      return indexer_impl<64, 128, 1>(d, s, q_idx, q_scale, w, k_idx, k_scale, row_begin,
                                      row_count, scores, ld, status, st, hist);
    return indexer_impl<64, 128, 4>(d, s, q_idx, q_scale, w, k_idx, k_scale, row_begin,
                                    row_count, scores, ld, status, st, hist);
  }
  return indexer_impl<4, 32, 64>(d, s, q_idx, q_scale, w, k_idx, k_scale, row_begin, row_count,
                                 scores, ld, status, st, nullptr);
}

// Indexer and top-k of rows [row_begin, row_begin + row_count) through a score slab, the
// indexer counting each row's first digit as it writes the scores (`hist`: row_count rows of
// kTopkBins words, zero on entry and zero again on return) when its shape allows.
dsa_status_t indexer_topk(const dsa_dims_t& d, const dsa_seqs_t& s, const uint8_t* q_idx,
                          const float* q_scale, const float* w, const uint8_t* k_idx,
                          const float* k_scale, int32_t row_begin, int32_t row_count,
                          float* slab, int64_t ld, uint32_t* hist, int32_t* idx, float* sel,
                          int32_t* status, cudaStream_t st) {
  uint32_t* h = indexer_counts_hist(d) ? hist : nullptr;
  dsa_status_t e = indexer_dispatch(d, s, q_idx, q_scale, w, k_idx, k_scale, row_begin,
                                    row_count, slab, ld, status, st, h);
  if (e != DSA_OK) return e;
  return topk_launch(d, s, slab, ld, row_begin, row_count, idx, status, st, h, sel);
}

// ------------------------------------------------------------------------ stage 2

// Cluster size and slice of the top-k launch for rows of up to `longest` keys: slices of at
// most 32768 keys (8 KB of bitmaps; 65536 when the launch has rows for two full waves, where
// fewer CTAs per row pay the per-CTA phases fewer times), then more CTAs per row while the rows
// alone leave SMs idle and slices stay at least 4096 keys long.  Longer rows than 8 slices take
// longer slices (larger bitmaps), as far as shared memory allows.
struct TopkShape {
  int csize;
  int slice;
};
TopkShape topk_shape(int64_t longest, int32_t row_count, int sm_count) {
  const int64_t max_slice = int64_t(row_count) >= 2 * int64_t(sm_count) ? 65536 : 32768;
  int c = 1;
  while (c < 8 && int64_t(c) * max_slice < longest) c *= 2;
  while (c < 8 && int64_t(row_count) * c < sm_count && int64_t(c) * 4096 < longest) c *= 2;
  const int64_t per = (ceil_div(std::max<int64_t>(1, longest), c) + 127) / 128 * 128;
  return TopkShape{c, static_cast<int>(std::min<int64_t>(per, INT32_MAX / 2))};
}

// `hist`: per-row first-digit histograms written with the scores (the fused indexer), or null
// (the top-k builds them itself).  `sel`: optional scores of the selected keys.
dsa_status_t topk_launch(const dsa_dims_t& d, const dsa_seqs_t& s, const float* scores, int64_t ld,
                         int32_t row_begin, int32_t row_count, int32_t* idx, int32_t* status,
                         cudaStream_t st, uint32_t* hist, float* sel) {
  if (row_count == 0) return DSA_OK;
  DeviceInfo info;
  if (device_info(&info) != DSA_OK) return DSA_ERR_CUDA;
  TopkParams prm{};
  prm.scores = scores;
  prm.ld = ld;
  prm.idx = idx;
  prm.sel = sel;
  prm.topk = d.topk;
  prm.decode = s.mode == DSA_DECODE;
  prm.row_begin = row_begin;
  prm.batch = s.batch;
  prm.cu_seqlens = s.cu_seqlens;
  prm.seq_lens = s.seq_lens;
  prm.max_seqlen = s.max_seqlen;
  prm.status = status;
  prm.hist = hist;
  const int64_t longest = std::min<int64_t>(max_keys(&s, row_begin, row_count), ld);
  const TopkShape shape = topk_shape(longest, row_count, info.sm_count);
  prm.csize = shape.csize;
  prm.slice = shape.slice;
  const int64_t smem = topk_smem_bytes(shape.slice);
  if (smem + 1024 > info.max_smem) return DSA_ERR_UNSUPPORTED_SHAPE;   // (+ static shared)
  if (prepare_kernel(dsa_topk_kernel, static_cast<int>(smem)) != DSA_OK) return DSA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(int64_t(row_count) * shape.csize));
  cfg.blockDim = dim3(kTopkThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = shape.csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // may launch while the previous kernel finishes (the kernel waits for it before any read)
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, dsa_topk_kernel, prm) != cudaSuccess) return DSA_ERR_CUDA;
  return launch_status();
}

// ------------------------------------------------------------------------ stage 3

size_t mla_ws_bytes(const dsa_dims_t& d, int splits, int32_t row_count) {
  if (splits <= 1) return 0;
  return size_t(splits) * row_count * d.h * (d.d_v + 1) * sizeof(float) + 256;
}

// Split-KV slices per decode row.  Only speed depends on the choice: one split needs no
// partials, so a cap on the partials' bytes (max_ws) always leaves a valid answer.
int mla_splits(const dsa_dims_t& d, const dsa_seqs_t& s, int32_t row_count, int sm_count,
               size_t max_ws = SIZE_MAX) {
  if (s.mode != DSA_DECODE || row_count <= 0) return 1;
  // Two CTAs (one per value half) per row and split; one CTA per SM.  Pick the split count
  // with the smallest estimated makespan: waves x (prologue + tiles per split), in tile units
  // (prologue ~3 tiles; a combine pass costs ~2 more).
  const int tiles = std::max(1, (std::min(d.topk, std::max(1, s.max_seqlen)) + 63) / 64);
  const int sms = std::max(1, sm_count);
  int best = 1;
  double best_t = 1e30;
  for (int sp = 1; sp <= std::min(16, std::max(1, tiles / 4)); ++sp) {
    if (mla_ws_bytes(d, sp, row_count) > max_ws) continue;
    const double waves = std::ceil(2.0 * row_count * sp / sms);
    const double t = waves * (3.0 + std::ceil(double(tiles) / sp)) + (sp > 1 ? 2.0 : 0.0);
    if (t < best_t - 1e-9) {
      best_t = t;
      best = sp;
    }
  }
  return best;
}

// The inputs and row geometry shared by the attention forward and the target pass.
MlaParams mla_params(const dsa_dims_t& d, const dsa_seqs_t& s, const uint16_t* q,
                     const uint16_t* kv, const int32_t* idx, int32_t row_begin, int32_t row_count,
                     int32_t splits, int32_t* status) {
  MlaParams prm{};
  prm.q = reinterpret_cast<const __nv_bfloat16*>(q);
  prm.kv = reinterpret_cast<const __nv_bfloat16*>(kv);
  prm.idx = idx;
  prm.row_begin = row_begin;
  prm.row_count = row_count;
  prm.topk = d.topk;
  prm.h = d.h;
  prm.splits = splits;
  prm.scale_log2 = d.softmax_scale * 1.4426950408889634f;
  prm.decode = s.mode == DSA_DECODE;
  prm.batch = s.batch;
  prm.cu_seqlens = s.cu_seqlens;
  prm.seq_lens = s.seq_lens;
  prm.block_table = s.block_table;
  prm.max_blocks = s.max_blocks;
  prm.kv_stride = s.max_seqlen;
  prm.max_seqlen = s.max_seqlen;
  prm.block_size = d.block_size > 0 ? d.block_size : 64;
  prm.num_kv_rows = s.num_kv_rows;
  prm.status = status;
  prm.ld_target = d.topk;
  return prm;
}

template <int D_QK, int D_V>
dsa_status_t mla_impl(const dsa_dims_t& d, const dsa_seqs_t& s, const uint16_t* q,
                      const uint16_t* kv, const int32_t* idx, int32_t row_begin, int32_t row_count,
                      uint16_t* out, float* lse, void* ws, size_t ws_bytes, int32_t* status,
                      cudaStream_t st, int splits) {
  using C = MlaCfg<D_QK, D_V>;
  MlaParams prm = mla_params(d, s, q, kv, idx, row_begin, row_count, splits, status);
  prm.out = reinterpret_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  if (splits > 1) {
    if (ws == nullptr || ws_bytes < mla_ws_bytes(d, splits, row_count))
      return DSA_ERR_WORKSPACE_TOO_SMALL;
    prm.part_o = static_cast<float*>(ws);
    prm.part_lse = prm.part_o + size_t(splits) * row_count * d.h * D_V;
  }
  // Q in 64-dim x 128-head boxes
  CUtensorMap q_map;
  if (make_row_map(&q_map, q, uint64_t(s.total_rows) * d.h, D_QK * 2, 128, 128) != DSA_OK)
    return DSA_ERR_CUDA;
  auto k = dsa_sparse_mla_kernel<D_QK, D_V>;
  if (prepare_kernel(k, C::SMEM_BYTES) != DSA_OK) return DSA_ERR_CUDA;
  if (launch_pdl(k, dim3(2 * row_count, splits), C::THREADS, C::SMEM_BYTES, st, q_map, prm) !=
      DSA_OK)
    return DSA_ERR_CUDA;
  if (splits > 1) {
    dsa_mla_combine_kernel<D_V><<<dim3(row_count, d.h), 128, 0, st>>>(prm);
    return launch_status();
  }
  return DSA_OK;
}

dsa_status_t mla_dispatch(const dsa_dims_t& d, const dsa_seqs_t& s, const uint16_t* q,
                          const uint16_t* kv, const int32_t* idx, int32_t row_begin,
                          int32_t row_count, uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                          int32_t* status, cudaStream_t st, int splits) {
  if (row_count == 0) return DSA_OK;
  if (d.d_qk == 576)
    return mla_impl<576, 512>(d, s, q, kv, idx, row_begin, row_count, out, lse, ws, ws_bytes,
                              status, st, splits);
  return mla_impl<160, 128>(d, s, q, kv, idx, row_begin, row_count, out, lse, ws, ws_bytes,
                            status, st, splits);
}

// ------------------------------------------------------------------------ dsa_forward plan

struct ForwardPlan {
  int64_t slab_floats = 0;   // score slab
  int64_t idx_ints = 0;      // chunk indices when idx_out is null
  int mla_splits = 1;
  size_t mla_bytes = 0;
  int64_t hist_rows = 0;     // first-digit histograms of one chunk's rows (fused indexer)
  size_t total = 0;
};

int64_t round4(int64_t x) { return (x + 3) / 4 * 4; }

// Prefill rows per chunk of a sequence of L rows: as many as the slab budget allows; when the
// sequence needs several chunks, a multiple of sm_count / 2 rows, so that each chunk's attention
// launch (two CTAs per row, one per SM) fills whole waves.
int64_t chunk_rows_for(int64_t L, int sm_count) {
  const int64_t ld = round4(L);
  const int64_t cap = std::max<int64_t>(1, int64_t(kSlabBudget / (ld * 4)));
  if (cap >= L) return L;
  const int64_t wave = std::max(1, sm_count / 2);
  return cap >= wave ? cap / wave * wave : cap;
}

ForwardPlan plan_forward(const dsa_dims_t& d, const dsa_seqs_t& s, int sm_count) {
  ForwardPlan p;
  if (s.mode == DSA_DECODE) {
    p.slab_floats = int64_t(s.batch) * round4(s.max_seqlen);
    p.idx_ints = int64_t(s.batch) * d.topk;
    p.mla_splits = mla_splits(d, s, s.batch, sm_count);
    p.mla_bytes = mla_ws_bytes(d, p.mla_splits, s.batch);
    p.hist_rows = s.batch;
  } else {
    const int32_t* cu = s.cu_seqlens_host;
    int64_t max_rows = 0;
    for (int b = 0; b < s.batch; ++b) {
      const int64_t L = cu[b + 1] - cu[b];
      if (L <= 0) continue;
      const int64_t rows = chunk_rows_for(L, sm_count);
      p.slab_floats = std::max(p.slab_floats, rows * round4(L));
      max_rows = std::max(max_rows, rows);
    }
    p.idx_ints = max_rows * d.topk;
    p.hist_rows = max_rows;
  }
  if (!indexer_counts_hist(d)) p.hist_rows = 0;
  auto align = [](size_t x) { return (x + 255) / 256 * 256; };
  p.total = align(p.slab_floats * 4) + align(p.idx_ints * 4) + align(p.mla_bytes) +
            size_t(p.hist_rows) * kTopkBins * 4;
  return p;
}

// ------------------------------------------------------------------------ indexer training

// Split count of the target pass: keys are independent there, so splits need no combine; fill
// the SMs when the rows alone do not, keeping at least two tiles per CTA pair.
int target_splits(const dsa_dims_t& d, int32_t row_count, int sm_count) {
  const int tiles = d.topk / 64;
  return std::max(1, std::min({16, tiles / 2, sm_count / std::max(1, 2 * row_count)}));
}

template <int D_QK, int D_V>
dsa_status_t target_impl(const dsa_dims_t& d, const dsa_seqs_t& s, const uint16_t* q,
                         const uint16_t* kv, const int32_t* idx, const float* lse,
                         int32_t row_begin, int32_t row_count, float* target, int64_t ld_target,
                         int32_t* status, cudaStream_t st, int sm_count) {
  using C = MlaCfg<D_QK, D_V>;
  const int splits = target_splits(d, row_count, sm_count);
  MlaParams prm = mla_params(d, s, q, kv, idx, row_begin, row_count, splits, status);
  prm.lse_in = lse;
  prm.target = target;
  prm.ld_target = ld_target;
  CUtensorMap q_map;
  if (make_row_map(&q_map, q, uint64_t(s.total_rows) * d.h, D_QK * 2, 128, 128) != DSA_OK)
    return DSA_ERR_CUDA;
  auto k = dsa_sparse_mla_kernel<D_QK, D_V, true>;
  if (prepare_kernel(k, C::SMEM_BYTES) != DSA_OK) return DSA_ERR_CUDA;
  k<<<dim3(2 * row_count, splits), C::THREADS, C::SMEM_BYTES, st>>>(q_map, prm);
  return launch_status();
}

// (64, 128): the tensor-core kernel; the small indexer shape (4 heads: too narrow an MMA N)
// runs on the CUDA cores.
dsa_status_t kl_backward_launch(bool full, const IdxBwdParams& prm, cudaStream_t st) {
  if (full) {
    auto k = dsa_indexer_kl_bwd_tc_kernel;
    if (prepare_kernel(k, KlTcCfg::SMEM_BYTES) != DSA_OK) return DSA_ERR_CUDA;
    k<<<prm.row_count, KlTcCfg::THREADS, KlTcCfg::SMEM_BYTES, st>>>(prm);
  } else {
    using C = IdxBwdCfg<4, 32>;
    auto k = dsa_indexer_kl_bwd_kernel<4, 32>;
    if (prepare_kernel(k, C::SMEM_BYTES) != DSA_OK) return DSA_ERR_CUDA;
    k<<<prm.row_count, C::THREADS, C::SMEM_BYTES, st>>>(prm);
  }
  return launch_status();
}

// ------------------------------------------------------------------------ dsa_forward body

// The whole path for query rows [w0, w1): the query-side pointers (q_idx, q_scale, w, q, out,
// lse, idx_out) are indexed by absolute row, the key-side ones (k_idx, k_scale, kv) by physical
// row.  Prefill: per sequence, the window's rows with at most topk prior keys run dense attention
// (when no indices are kept), the rest in chunks of indexer + top-k (fused first digit) +
// sparse attention.  Decode: the window's sequences in one chunk.
dsa_status_t forward_window(const dsa_dims_t& d, const dsa_seqs_t& s, int64_t w0, int64_t w1,
                            const uint8_t* q_idx, const float* q_scale, const float* w,
                            const uint8_t* k_idx, const float* k_scale, const uint16_t* q,
                            const uint16_t* kv, int32_t* idx_out, float* sel_out, uint16_t* out,
                            float* lse, void* workspace, size_t workspace_bytes,
                            int32_t* dev_status, cudaStream_t st) {
  dsa_status_t e;
  if (!indexer_shape_ok(d, s.mode) || !mla_shape_ok(d)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!q_idx || !q_scale || !w || !k_idx || !q || !kv || !out || !lse)
    return DSA_ERR_INVALID_ARG;
  if (sel_out != nullptr && idx_out == nullptr) return DSA_ERR_INVALID_ARG;
  if (k_scale == nullptr && !interleaved_ok(s)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(k_scale) || !aligned16(q) ||
      !aligned16(kv) || !aligned16(out) || !aligned16(lse) || !aligned16(idx_out) ||
      !aligned16(sel_out) || !aligned16(workspace) || !aligned16(q_scale) || !aligned16(w))
    return DSA_ERR_MISALIGNED;
  DeviceInfo info;
  if (device_info(&info) != DSA_OK) return DSA_ERR_CUDA;
  const ForwardPlan plan = plan_forward(d, s, info.sm_count);
  if (workspace == nullptr || workspace_bytes < plan.total) return DSA_ERR_WORKSPACE_TOO_SMALL;
  if (w1 <= w0) return DSA_OK;
  auto align = [](size_t x) { return (x + 255) / 256 * 256; };
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  float* slab = reinterpret_cast<float*>(wsb);
  int32_t* idx_ws = reinterpret_cast<int32_t*>(wsb + align(plan.slab_floats * 4));
  void* mla_ws = wsb + align(plan.slab_floats * 4) + align(plan.idx_ints * 4);
  uint32_t* hist = plan.hist_rows > 0
                       ? reinterpret_cast<uint32_t*>(wsb + align(plan.slab_floats * 4) +
                                                     align(plan.idx_ints * 4) +
                                                     align(plan.mla_bytes))
                       : nullptr;
  // the histograms start at zero; each top-k launch leaves its rows zeroed for the next chunk
  if (hist != nullptr &&
      cudaMemsetAsync(hist, 0, size_t(plan.hist_rows) * kTopkBins * 4, st) != cudaSuccess)
    return DSA_ERR_CUDA;

  if (s.mode == DSA_DECODE) {
    const int32_t rb = static_cast<int32_t>(w0), rc = static_cast<int32_t>(w1 - w0);
    // a window of fewer sequences may split more: as far as the planned partials allow
    const int splits = rc == s.batch ? plan.mla_splits
                                     : mla_splits(d, s, rc, info.sm_count, plan.mla_bytes);
    const size_t mla_bytes = mla_ws_bytes(d, splits, rc);
    if (idx_out == nullptr && s.max_seqlen <= d.topk)   // every context key is kept: dense
      return mla_dispatch(d, s, q, kv, nullptr, rb, rc, out, lse, mla_ws, mla_bytes, dev_status,
                          st, splits);
    const int64_t ld = round4(s.max_seqlen);
    int32_t* idx = idx_out ? idx_out + int64_t(rb) * d.topk : idx_ws;
    float* sel = sel_out ? sel_out + int64_t(rb) * d.topk : nullptr;
    if ((e = indexer_topk(d, s, q_idx, q_scale, w, k_idx, k_scale, rb, rc, slab, ld, hist, idx,
                          sel, dev_status, st)) != DSA_OK)
      return e;
    return mla_dispatch(d, s, q, kv, idx, rb, rc, out, lse, mla_ws, mla_bytes, dev_status, st,
                        splits);
  }
  const int32_t* cu = s.cu_seqlens_host;
  for (int b = 0; b < s.batch; ++b) {
    const int64_t L = cu[b + 1] - cu[b];
    // the window's rows of this sequence, as positions [p0, p1)
    const int64_t p0 = std::max<int64_t>(w0, cu[b]) - cu[b];
    const int64_t p1 = std::min<int64_t>(w1, cu[b + 1]) - cu[b];
    if (L <= 0 || p1 <= p0) continue;
    const int64_t ld = round4(p1);
    const int64_t rows = chunk_rows_for(L, info.sm_count);
    // rows with at most topk prior keys keep all of them: dense attention, no indexer or top-k
    // (unless the caller wants the indices)
    const int64_t dense_end = idx_out == nullptr ? std::min<int64_t>(p1, d.topk) : p0;
    if (dense_end > p0 &&
        (e = mla_dispatch(d, s, q, kv, nullptr, static_cast<int32_t>(cu[b] + p0),
                          static_cast<int32_t>(dense_end - p0), out, lse, nullptr, 0, dev_status,
                          st, 1)) != DSA_OK)
      return e;
    for (int64_t r0 = std::max(p0, dense_end); r0 < p1; r0 += rows) {
      const int32_t row_begin = static_cast<int32_t>(cu[b] + r0);
      const int32_t row_count = static_cast<int32_t>(std::min(rows, p1 - r0));
      int32_t* idx = idx_out ? idx_out + int64_t(row_begin) * d.topk : idx_ws;
      float* sel = sel_out ? sel_out + int64_t(row_begin) * d.topk : nullptr;
      if ((e = indexer_topk(d, s, q_idx, q_scale, w, k_idx, k_scale, row_begin, row_count,
                            slab, ld, hist, idx, sel, dev_status, st)) != DSA_OK)
        return e;
      if ((e = mla_dispatch(d, s, q, kv, idx, row_begin, row_count, out, lse, nullptr, 0,
                            dev_status, st, 1)) != DSA_OK)
        return e;
    }
  }
  return DSA_OK;
}

// ------------------------------------------------------------------- training entry bodies

dsa_status_t kl_target_impl(const dsa_dims_t& d, const dsa_seqs_t& s, const uint16_t* q,
                            const uint16_t* kv, const int32_t* idx, const float* lse,
                            int32_t row_begin, int32_t row_count, float* target,
                            int64_t ld_target, int32_t* status, cudaStream_t st) {
  if (!mla_shape_ok(d)) return DSA_ERR_UNSUPPORTED_SHAPE;
  dsa_status_t e;
  if ((e = check_rows(&s, row_begin, row_count)) != DSA_OK) return e;
  if (!q || !kv || !lse || !target) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(idx) || !aligned16(lse) || !aligned16(target))
    return DSA_ERR_MISALIGNED;
  if (row_count == 0) return DSA_OK;
  DeviceInfo info;
  if (device_info(&info) != DSA_OK) return DSA_ERR_CUDA;
  if (d.d_qk == 576)
    return target_impl<576, 512>(d, s, q, kv, idx, lse, row_begin, row_count, target, ld_target,
                                 status, st, info.sm_count);
  return target_impl<160, 128>(d, s, q, kv, idx, lse, row_begin, row_count, target, ld_target,
                               status, st, info.sm_count);
}

// idx NULL: dense mode (every prior key of each row, the caller checked the geometry)
dsa_status_t kl_backward_impl(const dsa_dims_t& d, const dsa_seqs_t& s, const uint8_t* q_idx,
                              const float* q_scale, const float* w, const uint8_t* k_idx,
                              const float* k_scale, const int32_t* idx, const float* sel,
                              const float* target,
                              int64_t ld_target, int32_t row_begin, int32_t row_count,
                              float* loss, float* dw, float* dq, float* dk, int32_t* status,
                              cudaStream_t st) {
  const bool full = d.h_idx == 64 && d.d_idx == 128;
  const bool tiny = d.h_idx == 4 && d.d_idx == 32;
  if (!full && !tiny) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (full && d.topk % KlTcCfg::BK != 0) return DSA_ERR_UNSUPPORTED_SHAPE;   // whole key tiles
  dsa_status_t e;
  if ((e = check_rows(&s, row_begin, row_count)) != DSA_OK) return e;
  if (!q_idx || !q_scale || !w || !k_idx || !k_scale || !target || !loss || !dw || !dq || !dk)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(idx) || !aligned16(target) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(q_scale) || !aligned16(w) ||
      !aligned16(k_scale) || !aligned16(loss) || !aligned16(dw))
    return DSA_ERR_MISALIGNED;
  if (row_count == 0) return DSA_OK;
  IdxBwdParams prm{};
  prm.q_idx = q_idx;
  prm.q_scale = q_scale;
  prm.w = w;
  prm.k_idx = k_idx;
  prm.k_scale = k_scale;
  prm.idx = idx;
  prm.target = target;
  prm.sel = idx != nullptr ? sel : nullptr;
  prm.ld_target = ld_target;
  prm.dense = idx == nullptr;
  prm.loss = loss;
  prm.dw = dw;
  prm.dq = dq;
  prm.dk = dk;
  prm.row_begin = row_begin;
  prm.row_count = row_count;
  prm.topk = d.topk;
  prm.decode = s.mode == DSA_DECODE;
  prm.batch = s.batch;
  prm.cu_seqlens = s.cu_seqlens;
  prm.seq_lens = s.seq_lens;
  prm.block_table = s.block_table;
  prm.max_blocks = s.max_blocks;
  prm.kv_stride = s.max_seqlen;
  prm.max_seqlen = s.max_seqlen;
  prm.block_size = d.block_size > 0 ? d.block_size : 64;
  prm.num_kv_rows = s.num_kv_rows;
  prm.status = status;
  return kl_backward_launch(full, prm, st);
}

// ---------------------------------------------------------------- bounded-wait self-test

// One CTA waits on an mbarrier that nothing arrives at, with the wait every kernel here uses
// (lane 0 polls, 2 s limit, then the whole warp gives up).  As in the kernels above, the first
// warp to give up raises the CTA's abort flag so that the other ends its wait early; each warp
// records a timeout in the status word and the CTA then exits normally.
__global__ void __launch_bounds__(64) dsa_selftest_wait_kernel(int32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (!warp_mbar_wait(smem_u32(&bar), 0, &abort_flag) && (threadIdx.x & 31) == 0) {
    abort_flag = 1;
    atomicOr(status, kStatusTimeout);
  }
}

// ------------------------------------------------------- distributed shared memory probe

// Each cluster of two CTAs (one per SM) exchanges `bytes` of its shared memory with its partner
// `reps` times over distributed shared memory: every thread stores 16-byte words into the
// partner's buffer (st.shared::cluster.v4), both CTAs at once, the traffic pattern of a logit
// exchange between the two CTAs of an attention row.  ns[cluster] = the exchange time of the
// cluster (%globaltimer between two cluster barriers, CTA 0); after the last round every CTA
// checks that its buffer holds its partner's last pattern and adds the mismatching words to *bad.
constexpr int kProbeThreads = 512;
__global__ void __launch_bounds__(kProbeThreads) dsa_probe_dsmem_kernel(int32_t bytes,
                                                                       int32_t reps,
                                                                       uint64_t* ns,
                                                                       int32_t* bad) {
  extern __shared__ __align__(16) uint8_t probe_smem[];
  uint4* buf = reinterpret_cast<uint4*>(probe_smem);
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int words = bytes / 16;
  const uint32_t dst = map_to_rank(smem_u32(buf), peer);
  cluster_sync();
  const uint64_t t0 = global_timer_ns();
  for (int r = 0; r < reps; ++r) {
    for (int j = threadIdx.x; j < words; j += kProbeThreads) {
      const uint32_t v = (uint32_t(r) << 20) ^ (uint32_t(j) << 1) ^ rank;
      asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + j * 16),
                   "r"(v), "r"(v + 1u), "r"(v + 2u), "r"(v + 3u)
                   : "memory");
    }
  }
  cluster_sync();
  const uint64_t t1 = global_timer_ns();
  if (rank == 0 && threadIdx.x == 0) ns[blockIdx.x / 2] = t1 - t0;
  int miss = 0;
  for (int j = threadIdx.x; j < words; j += kProbeThreads) {
    const uint32_t v = (uint32_t(reps - 1) << 20) ^ (uint32_t(j) << 1) ^ peer;
    const uint4 w = buf[j];
    miss += (w.x != v) + (w.y != v + 1u) + (w.z != v + 2u) + (w.w != v + 3u);
  }
  if (miss) atomicAdd(bad, miss);
  cluster_sync();   // no CTA leaves while its partner may still read nothing of it (symmetry)
}

// ------------------------------------------------------- key-page stream probe

// Reads the pages of an interleaved indexer key cache (each page 64 key rows of d_idx bytes,
// then their 64 fp32 scales) into shared memory exactly as the decode indexer's producer does
// (one 3-D TMA box for the rows and a 256-byte bulk copy for the scales, both evict-first) and
// computes nothing: the read rate of the indexer's key stream with no arithmetic and no
// consumer, the practical ceiling of that access pattern.  CTA c takes a contiguous range of
// the page ids, as an indexer CTA takes a range of one row's pages; its warp loads 32 ids at a
// time and lane 0 issues their copies into a ring of `slots` page buffers.  An id outside
// [0, n_blocks) is skipped and counted in *bad, and so is a CTA whose bounded wait ran out (it
// then stops issuing and waits, again bounded, for the copies in flight).
constexpr int kStreamMaxSlots = 32;
__global__ void __launch_bounds__(32) dsa_probe_stream_kernel(
    const __grid_constant__ CUtensorMap kmap, const uint8_t* k_blocks, const int32_t* ids,
    int64_t n_ids, int64_t n_blocks, int32_t d_idx, int32_t slots, int32_t* bad) {
  extern __shared__ uint8_t stream_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(stream_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[kStreamMaxSlots];
  const int lane = threadIdx.x;
  const uint32_t key_bytes = 64u * static_cast<uint32_t>(d_idx);
  const int64_t page_bytes = key_bytes + 256;
  const uint32_t slot_bytes = (key_bytes + 256u + 1023u) & ~1023u;   // swizzle-atom aligned
  const int64_t per = (n_ids + gridDim.x - 1) / gridDim.x;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * per;
  const int64_t i1 = i0 + per < n_ids ? i0 + per : n_ids;
  uint64_t pol = 0;
  if (lane == 0) {
    for (int s = 0; s < slots; ++s) mbar_init(smem_u32(&bars[s]), 1);
    fence_mbar_init();
    tma_prefetch_desc(&kmap);
    pol = l2_evict_first();
  }
  __syncwarp();
  int issued = 0, miss = 0, ok = 1;
  for (int64_t c0 = i0; c0 < i1 && ok; c0 += 32) {
    const int64_t mine = c0 + lane < i1 ? ids[c0 + lane] : 0;
    const int cnt = i1 - c0 < 32 ? static_cast<int>(i1 - c0) : 32;
    for (int j = 0; j < cnt; ++j) {
      const int64_t id = __shfl_sync(0xffffffffu, mine, j);
      if (lane != 0 || !ok) continue;
      if (id < 0 || id >= n_blocks) {
        ++miss;
        continue;
      }
      const int s = issued % slots;
      if (issued >= slots &&
          !mbar_wait(smem_u32(&bars[s]), ((issued / slots) - 1) & 1, nullptr)) {
        ok = 0;
        continue;
      }
      const uint32_t dst = smem_u32(ring + static_cast<size_t>(s) * slot_bytes);
      mbar_arrive_expect_tx(smem_u32(&bars[s]), key_bytes + 256u);
      tma_load_3d_hint(dst, &kmap, smem_u32(&bars[s]), 0, 0, static_cast<int32_t>(id), pol);
      bulk_load_g2s_hint(dst + key_bytes, k_blocks + id * page_bytes + key_bytes, 256u,
                         smem_u32(&bars[s]), pol);
      ++issued;
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
  }
  if (lane != 0) return;
  // never leave a copy in flight into the shared memory of an exiting CTA
  for (int k = max(0, issued - slots); k < issued; ++k)
    if (!mbar_wait(smem_u32(&bars[k % slots]), (k / slots) & 1, nullptr)) ok = 0;
  if (!ok) ++miss;
  if (miss) atomicAdd(bad, miss);
}

}  // namespace

// ============================================================================ C ABI

extern "C" {

int32_t dsa_abi_version(void) { return DSA_ABI_VERSION; }

const char* dsa_status_string(dsa_status_t st) {
  switch (st) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case DSA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case DSA_ERR_MISALIGNED: return "misaligned pointer or leading dimension";
    case DSA_ERR_BAD_INDEX: return "index outside the caches";
    case DSA_ERR_TIMEOUT: return "device wait timed out";
    case DSA_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

dsa_status_t dsa_indexer_scores(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                const uint8_t* q_idx, const float* q_scale, const float* w,
                                const uint8_t* k_idx, const float* k_scale, int32_t row_begin,
                                int32_t row_count, float* scores, int64_t ld_scores,
                                uint32_t* hist, int32_t* dev_status, dsa_stream_t stream) {
  NvtxRange nvtx_range("dsa_indexer_scores");
  dsa_status_t e = check_common(dims, seqs);
  if (e != DSA_OK) return e;
  if (!indexer_shape_ok(*dims, seqs->mode)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (hist != nullptr && !indexer_counts_hist(*dims)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if ((e = check_rows(seqs, row_begin, row_count)) != DSA_OK) return e;
  if (!q_idx || !q_scale || !w || !k_idx || !scores) return DSA_ERR_INVALID_ARG;
  if (k_scale == nullptr && !interleaved_ok(*seqs)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(k_scale) || !aligned16(scores) ||
      !aligned16(hist) || ld_scores % 4 != 0)
    return DSA_ERR_MISALIGNED;
  if (ld_scores < max_keys(seqs, row_begin, row_count)) return DSA_ERR_INVALID_ARG;
  return indexer_dispatch(*dims, *seqs, q_idx, q_scale, w, k_idx, k_scale, row_begin, row_count,
                          scores, ld_scores, dev_status, reinterpret_cast<cudaStream_t>(stream),
                          hist);
}

dsa_status_t dsa_topk(const dsa_dims_t* dims, const dsa_seqs_t* seqs, const float* scores,
                      int64_t ld_scores, uint32_t* hist, int32_t row_begin, int32_t row_count,
                      int32_t* idx, float* sel_out, int32_t* dev_status, dsa_stream_t stream) {
  NvtxRange nvtx_range("dsa_topk");
  dsa_status_t e = check_common(dims, seqs);
  if (e != DSA_OK) return e;
  if ((e = check_rows(seqs, row_begin, row_count)) != DSA_OK) return e;
  if (!scores || !idx) return DSA_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(idx) || !aligned16(hist) || !aligned16(sel_out) ||
      ld_scores % 4 != 0)
    return DSA_ERR_MISALIGNED;
  if (ld_scores < max_keys(seqs, row_begin, row_count)) return DSA_ERR_INVALID_ARG;
  return topk_launch(*dims, *seqs, scores, ld_scores, row_begin, row_count, idx, dev_status,
                     reinterpret_cast<cudaStream_t>(stream), hist, sel_out);
}

size_t dsa_indexer_topk_workspace_size(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                       int32_t row_count) {
  if (check_common(dims, seqs) != DSA_OK || row_count < 0) return 0;
  const size_t slab = size_t(row_count) * size_t(round4(seqs->max_seqlen)) * 4;
  return (slab + 255) / 256 * 256 + size_t(row_count) * kTopkBins * 4;
}

dsa_status_t dsa_indexer_topk(const dsa_dims_t* dims, const dsa_seqs_t* seqs, const uint8_t* q_idx,
                              const float* q_scale, const float* w, const uint8_t* k_idx,
                              const float* k_scale, int32_t row_begin, int32_t row_count,
                              int32_t* idx, float* sel_out, void* workspace,
                              size_t workspace_bytes, int32_t* dev_status, dsa_stream_t stream) {
  NvtxRange nvtx_range("dsa_indexer_topk");
  dsa_status_t e = check_common(dims, seqs);
  if (e != DSA_OK) return e;
  if (!indexer_shape_ok(*dims, seqs->mode)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if ((e = check_rows(seqs, row_begin, row_count)) != DSA_OK) return e;
  if (!q_idx || !q_scale || !w || !k_idx || !idx) return DSA_ERR_INVALID_ARG;
  if (k_scale == nullptr && !interleaved_ok(*seqs)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(k_scale) || !aligned16(idx) ||
      !aligned16(sel_out) || !aligned16(workspace))
    return DSA_ERR_MISALIGNED;
  if (row_count == 0) return DSA_OK;
  const size_t need = dsa_indexer_topk_workspace_size(dims, seqs, row_count);
  if (workspace == nullptr || workspace_bytes < need) return DSA_ERR_WORKSPACE_TOO_SMALL;
  const int64_t ld = round4(max_keys(seqs, row_begin, row_count));
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  float* slab = reinterpret_cast<float*>(wsb);
  uint32_t* hist = reinterpret_cast<uint32_t*>(
      wsb + (size_t(row_count) * size_t(round4(seqs->max_seqlen)) * 4 + 255) / 256 * 256);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (indexer_counts_hist(*dims) &&
      cudaMemsetAsync(hist, 0, size_t(row_count) * kTopkBins * 4, st) != cudaSuccess)
    return DSA_ERR_CUDA;
  return indexer_topk(*dims, *seqs, q_idx, q_scale, w, k_idx, k_scale, row_begin, row_count, slab,
                      ld, hist, idx, sel_out, dev_status, st);
}

size_t dsa_sparse_mla_workspace_size(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                     int32_t row_count) {
  if (check_common(dims, seqs) != DSA_OK) return 0;
  DeviceInfo info;
  if (device_info(&info) != DSA_OK) return 0;
  return mla_ws_bytes(*dims, mla_splits(*dims, *seqs, row_count, info.sm_count), row_count);
}

dsa_status_t dsa_sparse_mla_fwd(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                                int32_t row_begin, int32_t row_count, uint16_t* out, float* lse,
                                void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                dsa_stream_t stream) {
  NvtxRange nvtx_range("dsa_sparse_mla_fwd");
  dsa_status_t e = check_common(dims, seqs);
  if (e != DSA_OK) return e;
  if (!mla_shape_ok(*dims)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if ((e = check_rows(seqs, row_begin, row_count)) != DSA_OK) return e;
  if (!q || !kv || !out || !lse) return DSA_ERR_INVALID_ARG;
  if (idx == nullptr && !dense_ok(*dims, seqs, row_begin, row_count)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(idx) || !aligned16(out) || !aligned16(lse) ||
      !aligned16(workspace))
    return DSA_ERR_MISALIGNED;
  DeviceInfo info;
  if (device_info(&info) != DSA_OK) return DSA_ERR_CUDA;
  const int splits = mla_splits(*dims, *seqs, row_count, info.sm_count);
  return mla_dispatch(*dims, *seqs, q, kv, idx, row_begin, row_count, out, lse, workspace,
                      workspace_bytes, dev_status, reinterpret_cast<cudaStream_t>(stream), splits);
}

size_t dsa_sparse_mla_workspace_size_for(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                         int32_t row_count, int32_t sm_count, size_t max_bytes) {
  if (check_common(dims, seqs) != DSA_OK || sm_count <= 0 || row_count < 0) return 0;
  return mla_ws_bytes(*dims, mla_splits(*dims, *seqs, row_count, sm_count, max_bytes), row_count);
}

size_t dsa_forward_workspace_size_for(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                      int32_t sm_count) {
  if (check_common(dims, seqs) != DSA_OK || sm_count <= 0) return 0;
  return plan_forward(*dims, *seqs, sm_count).total;
}

int32_t dsa_forward_chunk_rows_for(const dsa_dims_t* dims, const dsa_seqs_t* seqs, int32_t seq,
                                   int32_t sm_count) {
  if (check_common(dims, seqs) != DSA_OK || sm_count <= 0) return 0;
  if (seqs->mode != DSA_PREFILL) return seqs->batch;
  if (seq < 0 || seq >= seqs->batch) return 0;
  const int64_t L = seqs->cu_seqlens_host[seq + 1] - seqs->cu_seqlens_host[seq];
  return L <= 0 ? 0 : static_cast<int32_t>(chunk_rows_for(L, sm_count));
}

size_t dsa_forward_workspace_size(const dsa_dims_t* dims, const dsa_seqs_t* seqs) {
  if (check_common(dims, seqs) != DSA_OK) return 0;
  DeviceInfo info;
  if (device_info(&info) != DSA_OK) return 0;
  return plan_forward(*dims, *seqs, info.sm_count).total;
}

dsa_status_t dsa_forward(const dsa_dims_t* dims, const dsa_seqs_t* seqs, const uint8_t* q_idx,
                         const float* q_scale, const float* w, const uint8_t* k_idx,
                         const float* k_scale, const uint16_t* q, const uint16_t* kv,
                         int32_t* idx_out, float* sel_out, uint16_t* out, float* lse,
                         void* workspace, size_t workspace_bytes, int32_t* dev_status,
                         dsa_stream_t stream) {
  NvtxRange nvtx_range("dsa_forward");
  dsa_status_t e = check_common(dims, seqs);
  if (e != DSA_OK) return e;
  return forward_window(*dims, *seqs, 0, seqs->total_rows, q_idx, q_scale, w, k_idx, k_scale, q,
                        kv, idx_out, sel_out, out, lse, workspace, workspace_bytes, dev_status,
                        reinterpret_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_forward_rows(const dsa_dims_t* dims, const dsa_seqs_t* seqs, int32_t row_begin,
                              int32_t row_count, const uint8_t* q_idx, const float* q_scale,
                              const float* w, const uint8_t* k_idx, const float* k_scale,
                              const uint16_t* q, const uint16_t* kv, int32_t* idx_out,
                              float* sel_out, uint16_t* out, float* lse, void* workspace,
                              size_t workspace_bytes, int32_t* dev_status, dsa_stream_t stream) {
  NvtxRange nvtx_range("dsa_forward_rows");
  dsa_status_t e = check_common(dims, seqs);
  if (e != DSA_OK) return e;
  if ((e = check_rows(seqs, row_begin, row_count)) != DSA_OK) return e;
  if (!q_idx || !q_scale || !w || !q || !out || !lse) return DSA_ERR_INVALID_ARG;
  const dsa_dims_t& d = *dims;
  // the query-side arrays hold rows [row_begin, row_begin + row_count); the kernels index them
  // by absolute row, so they get bases moved back by row_begin rows (computed as integers; only
  // the caller's rows are ever addressed from them)
  auto back = [&](const void* p, size_t row_bytes) -> uintptr_t {
    return reinterpret_cast<uintptr_t>(p) - uintptr_t(row_begin) * row_bytes;
  };
  const size_t hi = size_t(d.h_idx);
  const uintptr_t q_idx_a = back(q_idx, hi * d.d_idx);
  const uintptr_t q_scale_a = back(q_scale, hi * 4);
  const uintptr_t w_a = back(w, hi * 4);
  const uintptr_t q_a = back(q, size_t(d.h) * d.d_qk * 2);
  const uintptr_t out_a = back(out, size_t(d.h) * d.d_v * 2);
  const uintptr_t lse_a = back(lse, size_t(d.h) * 4);
  const uintptr_t idx_a = idx_out ? back(idx_out, size_t(d.topk) * 4) : 0;
  const uintptr_t sel_a = sel_out ? back(sel_out, size_t(d.topk) * 4) : 0;
  return forward_window(d, *seqs, row_begin, row_begin + row_count,
                        reinterpret_cast<const uint8_t*>(q_idx_a),
                        reinterpret_cast<const float*>(q_scale_a),
                        reinterpret_cast<const float*>(w_a), k_idx, k_scale,
                        reinterpret_cast<const uint16_t*>(q_a), kv,
                        reinterpret_cast<int32_t*>(idx_a), reinterpret_cast<float*>(sel_a),
                        reinterpret_cast<uint16_t*>(out_a), reinterpret_cast<float*>(lse_a),
                        workspace, workspace_bytes, dev_status,
                        reinterpret_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_cache_append(const dsa_dims_t* dims, const dsa_seqs_t* seqs, const float* k_new,
                              const uint16_t* kv_new, uint8_t* k_cache, float* k_scale_cache,
                              uint16_t* kv_cache, int32_t* dev_status, dsa_stream_t stream) {
  NvtxRange nvtx_range("dsa_cache_append");
  dsa_status_t e = check_common(dims, seqs);
  if (e != DSA_OK) return e;
  const dsa_dims_t& d = *dims;
  const dsa_seqs_t& s = *seqs;
  if (s.mode != DSA_DECODE) return DSA_ERR_INVALID_ARG;
  const bool full = d.d_idx == 128 && d.d_qk == 576;
  const bool tiny = d.d_idx == 32 && d.d_qk == 160;
  if (!full && !tiny) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!k_new || !kv_new || !k_cache || !kv_cache) return DSA_ERR_INVALID_ARG;
  if (k_scale_cache == nullptr && !interleaved_ok(s)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(kv_new) || !aligned16(k_cache) ||
      !aligned16(k_scale_cache) || !aligned16(kv_cache))
    return DSA_ERR_MISALIGNED;
  AppendParams prm{};
  prm.k_new = k_new;
  prm.kv_new = reinterpret_cast<const uint4*>(kv_new);
  prm.k_cache = k_cache;
  prm.k_scale = k_scale_cache;
  prm.kv_cache = reinterpret_cast<uint4*>(kv_cache);
  prm.seq_lens = s.seq_lens;
  prm.block_table = s.block_table;
  prm.batch = s.batch;
  prm.max_blocks = s.max_blocks;
  prm.max_seqlen = s.max_seqlen;
  prm.block_size = d.block_size;
  prm.num_kv_rows = s.num_kv_rows;
  prm.status = dev_status;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid(static_cast<unsigned>(ceil_div(s.batch, 4)));
  if (full)
    dsa_cache_append_kernel<128, 576><<<grid, 128, 0, st>>>(prm);
  else
    dsa_cache_append_kernel<32, 160><<<grid, 128, 0, st>>>(prm);
  return launch_status();
}

dsa_status_t dsa_indexer_kl_target(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                   const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                                   const float* lse, int32_t row_begin, int32_t row_count,
                                   float* target, int32_t* dev_status, dsa_stream_t stream) {
  NvtxRange nvtx_range("dsa_indexer_kl_target");
  dsa_status_t e = check_common(dims, seqs);
  if (e != DSA_OK) return e;
  if (idx == nullptr && !dense_target_ok(*dims, seqs, row_begin, row_count))
    return DSA_ERR_INVALID_ARG;
  return kl_target_impl(*dims, *seqs, q, kv, idx, lse, row_begin, row_count, target, dims->topk,
                        dev_status, reinterpret_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_indexer_kl_target_dense(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                         const uint16_t* q, const uint16_t* kv, const float* lse,
                                         int32_t row_begin, int32_t row_count, float* target,
                                         int64_t ld_target, int32_t* dev_status,
                                         dsa_stream_t stream) {
  NvtxRange nvtx_range("dsa_indexer_kl_target_dense");
  dsa_status_t e = check_common(dims, seqs);
  if (e != DSA_OK) return e;
  if (seqs->mode != DSA_PREFILL) return DSA_ERR_INVALID_ARG;
  if ((e = check_rows(seqs, row_begin, row_count)) != DSA_OK) return e;
  if (ld_target % 64 != 0) return DSA_ERR_MISALIGNED;
  if (ld_target < (max_keys(seqs, row_begin, row_count) + 63) / 64 * 64 || ld_target < dims->topk)
    return DSA_ERR_INVALID_ARG;
  return kl_target_impl(*dims, *seqs, q, kv, nullptr, lse, row_begin, row_count, target,
                        ld_target, dev_status, reinterpret_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_indexer_kl_backward(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                     const uint8_t* q_idx, const float* q_scale, const float* w,
                                     const uint8_t* k_idx, const float* k_scale,
                                     const int32_t* idx, const float* sel_scores,
                                     const float* target, int32_t row_begin, int32_t row_count,
                                     float* loss, float* dw, float* dq, float* dk,
                                     int32_t* dev_status, dsa_stream_t stream) {
  NvtxRange nvtx_range("dsa_indexer_kl_backward");
  dsa_status_t e = check_common(dims, seqs);
  if (e != DSA_OK) return e;
  if (idx == nullptr) return DSA_ERR_INVALID_ARG;
  if (!aligned16(sel_scores)) return DSA_ERR_MISALIGNED;
  return kl_backward_impl(*dims, *seqs, q_idx, q_scale, w, k_idx, k_scale, idx, sel_scores,
                          target, dims->topk, row_begin, row_count, loss, dw, dq, dk, dev_status,
                          reinterpret_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_indexer_kl_backward_dense(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                           const uint8_t* q_idx, const float* q_scale,
                                           const float* w, const uint8_t* k_idx,
                                           const float* k_scale, const float* target,
                                           int64_t ld_target, int32_t row_begin,
                                           int32_t row_count, float* loss, float* dw, float* dq,
                                           float* dk, int32_t* dev_status, dsa_stream_t stream) {
  NvtxRange nvtx_range("dsa_indexer_kl_backward_dense");
  dsa_status_t e = check_common(dims, seqs);
  if (e != DSA_OK) return e;
  if (seqs->mode != DSA_PREFILL) return DSA_ERR_INVALID_ARG;
  if ((e = check_rows(seqs, row_begin, row_count)) != DSA_OK) return e;
  if (ld_target % 4 != 0) return DSA_ERR_MISALIGNED;
  const int64_t longest = max_keys(seqs, row_begin, row_count);
  if (ld_target < longest) return DSA_ERR_INVALID_ARG;
  // the CUDA-core kernel of the small shape keeps every entry in shared memory
  if (dims->h_idx == 4 && longest > IdxBwdCfg<4, 32>::MAX_K) return DSA_ERR_UNSUPPORTED_SHAPE;
  return kl_backward_impl(*dims, *seqs, q_idx, q_scale, w, k_idx, k_scale, nullptr, nullptr,
                          target, ld_target, row_begin, row_count, loss, dw, dq, dk, dev_status,
                          reinterpret_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_selftest_wait_timeout(int32_t* dev_status, dsa_stream_t stream) {
  if (dev_status == nullptr) return DSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    return DSA_ERR_MISALIGNED;
  dsa_selftest_wait_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(dev_status);
  return launch_status();
}

dsa_status_t dsa_probe_dsmem(int32_t clusters, int32_t bytes, int32_t reps, uint64_t* ns,
                             int32_t* bad, dsa_stream_t stream) {
  if (clusters <= 0 || reps <= 0 || bytes <= 0 || bytes % 16 != 0 || !ns || !bad)
    return DSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ns) & 7u) != 0 || (reinterpret_cast<uintptr_t>(bad) & 3u) != 0)
    return DSA_ERR_MISALIGNED;
  DeviceInfo info;
  if (device_info(&info) != DSA_OK) return DSA_ERR_CUDA;
  // at least 116 KB each, so that one CTA runs per SM: the two CTAs of a pair sit on two SMs
  const int smem = std::max(bytes, 116 * 1024);
  if (smem > info.max_smem - 1024) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (prepare_kernel(dsa_probe_dsmem_kernel, smem) != DSA_OK) return DSA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
  cfg.blockDim = dim3(kProbeThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, dsa_probe_dsmem_kernel, bytes, reps, ns, bad) != cudaSuccess)
    return DSA_ERR_CUDA;
  return launch_status();
}

dsa_status_t dsa_probe_page_stream(const void* k_blocks, const int32_t* block_ids,
                                   int64_t n_ids, int64_t n_blocks, int32_t d_idx,
                                   int32_t ctas_per_sm, int32_t* bad, dsa_stream_t stream) {
  if (!k_blocks || !block_ids || !bad || n_ids <= 0 || n_blocks <= 0 ||
      n_blocks > INT32_MAX || (d_idx != 32 && d_idx != 128) || ctas_per_sm < 1 ||
      ctas_per_sm > 8)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(k_blocks) || (reinterpret_cast<uintptr_t>(block_ids) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(bad) & 3u) != 0)
    return DSA_ERR_MISALIGNED;
  DeviceInfo info;
  if (device_info(&info) != DSA_OK) return DSA_ERR_CUDA;
  // the SM's shared memory split over its CTAs (1 KB of each reserved by the hardware, the
  // barriers static, 1 KB of alignment slack)
  const int64_t slot_bytes = (64 * d_idx + 256 + 1023) / 1024 * 1024;
  const int64_t budget = (int64_t(info.max_smem) + 1024) / ctas_per_sm - 1024 - 512 - 1024;
  const int64_t slots = std::min<int64_t>(kStreamMaxSlots, budget / slot_bytes);
  if (slots < 2) return DSA_ERR_UNSUPPORTED_SHAPE;
  const int smem = static_cast<int>(slots * slot_bytes + 1024);
  CUtensorMap kmap;
  if (make_block_map(&kmap, k_blocks, uint64_t(n_blocks), uint32_t(d_idx)) != DSA_OK)
    return DSA_ERR_CUDA;
  if (prepare_kernel(dsa_probe_stream_kernel, smem) != DSA_OK) return DSA_ERR_CUDA;
  const int64_t grid = std::min<int64_t>(int64_t(info.sm_count) * ctas_per_sm, n_ids);
  dsa_probe_stream_kernel<<<static_cast<unsigned>(grid), 32, smem,
                            reinterpret_cast<cudaStream_t>(stream)>>>(
      kmap, static_cast<const uint8_t*>(k_blocks), block_ids, n_ids, n_blocks, d_idx,
      static_cast<int32_t>(slots), bad);
  return launch_status();
}

dsa_status_t dsa_read_device_status(const int32_t* dev_status, dsa_stream_t stream,
                                    int32_t* raw) {
  if (dev_status == nullptr) return DSA_ERR_INVALID_ARG;
  int32_t v = 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&v, dev_status, sizeof v, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (raw) *raw = v;
  if (v & DSA_DEVICE_TIMEOUT) return DSA_ERR_TIMEOUT;
  if (v & DSA_DEVICE_BAD_INDEX) return DSA_ERR_BAD_INDEX;
  return DSA_OK;
}

// ---------------------------------------------------------------------------- no allocation
// Scratch for dsa_sparse_mla_fwd_noalloc: a device array built into the library.  In host code
// `g_noalloc_scratch` is only a stand-in symbol, never a device address; the address of each
// device's copy comes from cudaGetSymbolAddress with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DSA_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_ptr[kMaxDevices];

dsa_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return DSA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return DSA_OK;
}
}  // namespace

dsa_status_t dsa_sparse_mla_fwd_noalloc(const dsa_dims_t* dims, const dsa_seqs_t* seqs,
                                        const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                                        int32_t row_begin, int32_t row_count, uint16_t* out,
                                        float* lse, int32_t* dev_status, dsa_stream_t stream) {
  NvtxRange nvtx_range("dsa_sparse_mla_fwd_noalloc");
  dsa_status_t e = check_common(dims, seqs);
  if (e != DSA_OK) return e;
  if (!mla_shape_ok(*dims)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if ((e = check_rows(seqs, row_begin, row_count)) != DSA_OK) return e;
  if (!q || !kv || !out || !lse) return DSA_ERR_INVALID_ARG;
  if (idx == nullptr && !dense_ok(*dims, seqs, row_begin, row_count)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(idx) || !aligned16(out) || !aligned16(lse))
    return DSA_ERR_MISALIGNED;
  DeviceInfo info;
  if (device_info(&info) != DSA_OK) return DSA_ERR_CUDA;
  // the fastest split count whose partials fit the built-in array (one split needs none)
  const int splits =
      mla_splits(*dims, *seqs, row_count, info.sm_count, DSA_NOALLOC_SCRATCH_BYTES);
  const size_t need = mla_ws_bytes(*dims, splits, row_count);
  if (need > DSA_NOALLOC_SCRATCH_BYTES) return DSA_ERR_WORKSPACE_TOO_SMALL;   // unreachable
  void* scratch = nullptr;
  if (need > 0 && (e = noalloc_scratch(&scratch)) != DSA_OK) return e;
  return mla_dispatch(*dims, *seqs, q, kv, idx, row_begin, row_count, out, lse, scratch,
                      need > 0 ? DSA_NOALLOC_SCRATCH_BYTES : 0, dev_status,
                      reinterpret_cast<cudaStream_t>(stream), splits);
}

}  // extern "C"
