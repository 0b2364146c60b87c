// Decode cache append: the step upstream of the indexer.  Each decode sequence b has one new
// token at position p = seq_lens[b] - 1.  Its indexer key k_new[b] (fp32, D_I values) is
// quantised with one scale per token (scale = amax / 448 in fp32, 1 when amax = 0; codes =
// the e4m3 value nearest to x / scale, ties to even, saturating at +-448) and written with its
// scale, and its latent row kv_new[b] (bf16, D_QK values) is copied, at the physical row
// block_table[b][p / bs] * bs + p % bs (row b * max_seqlen + p without a block table).  The
// caches it fills are the indexer's "FP8 index" keys and the latent rows the sparse attention
// gathers ("FP8 index -> top-k selection -> sparse core attention", "DeepSeek V3.2-Exp Cuts
// Long-Context Costs with DeepSeek Sparse Attention (DSA)", pipeline summary).
//
// One warp per sequence: the key row is read with one float4 per lane (D_I = 128) and reduced
// to its max with warp shuffles; the latent row moves as 16-byte chunks.  An entry whose
// position or block falls outside the caches is skipped and reported.  The key cache may hold
// each 64-row block's scales right after its key rows (paged decode, no separate scale array).
#pragma once
#include <cuda_fp8.h>

#include "sm100.cuh"

namespace dsa {

struct AppendParams {
  const float* k_new;          // [batch, D_I]
  const uint4* kv_new;         // [batch, D_QK] bf16, as 16-byte chunks
  uint8_t* k_cache;            // [num_kv_rows, D_I] e4m3, or with k_scale null interleaved
                               // blocks: [num_kv_rows / 64][64 * D_I bytes | 64 fp32 scales]
  float* k_scale;              // [num_kv_rows] or null
  uint4* kv_cache;             // [num_kv_rows, D_QK] bf16, as 16-byte chunks
  const int32_t* seq_lens;     // [batch]
  const int32_t* block_table;  // [batch, max_blocks] or null
  int32_t batch, max_blocks, max_seqlen, block_size;
  int64_t num_kv_rows;
  int32_t* status;
};

template <int D_I, int D_QK>
__global__ void __launch_bounds__(128) dsa_cache_append_kernel(const AppendParams p) {
  static_assert(D_I % 32 == 0 && (D_QK * 2) % 16 == 0, "row sizes");
  const int b = blockIdx.x * 4 + static_cast<int>(threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= p.batch) return;                       // warp-uniform
  const int pos = p.seq_lens[b] - 1;
  bool ok = pos >= 0 && pos < p.max_seqlen;
  int64_t row = -1;
  if (ok) {
    if (p.block_table != nullptr) {
      const int64_t blk = p.block_table[static_cast<int64_t>(b) * p.max_blocks + pos / p.block_size];
      ok = blk >= 0 && (blk + 1) * p.block_size <= p.num_kv_rows;
      row = blk * p.block_size + pos % p.block_size;
    } else {
      row = static_cast<int64_t>(b) * p.max_seqlen + pos;
      ok = row < p.num_kv_rows;
    }
  }
  if (!ok) {
    if (lane == 0 && p.status) atomicOr(p.status, kStatusBadIndex);
    return;
  }
  // ---- indexer key: per-token scale and e4m3 codes
  constexpr int PER = D_I / 32;
  float x[PER];
  const float* src = p.k_new + static_cast<int64_t>(b) * D_I + lane * PER;
  if constexpr (PER == 4) {
    const float4 v = *reinterpret_cast<const float4*>(src);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  } else {
#pragma unroll
    for (int i = 0; i < PER; ++i) x[i] = src[i];
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = amax > 0.f ? amax / 448.f : 1.f;
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const float y = fminf(fmaxf(x[i] / scale, -448.f), 448.f);
    const uint32_t c = __nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3);
    packed |= c << (8 * i);
  }
  // the key row and its scale: separate arrays, or inside the row's 64-row block
  const int64_t blk = row / 64, r64 = row % 64;
  uint8_t* krow = p.k_scale != nullptr ? p.k_cache + row * D_I
                                       : p.k_cache + blk * (64 * (D_I + 4)) + r64 * D_I;
  float* sdst = p.k_scale != nullptr
                    ? p.k_scale + row
                    : reinterpret_cast<float*>(p.k_cache + blk * (64 * (D_I + 4)) + 64 * D_I) + r64;
  uint8_t* kdst = krow + lane * PER;
  if constexpr (PER == 4) {
    *reinterpret_cast<uint32_t*>(kdst) = packed;
  } else {
#pragma unroll
    for (int i = 0; i < PER; ++i) kdst[i] = static_cast<uint8_t>(packed >> (8 * i));
  }
  if (lane == 0) *sdst = scale;
  // ---- latent row
  constexpr int CHUNKS = D_QK * 2 / 16;
  const uint4* ksrc = p.kv_new + static_cast<int64_t>(b) * CHUNKS;
  uint4* kvdst = p.kv_cache + row * CHUNKS;
  for (int c = lane; c < CHUNKS; c += 32) kvdst[c] = ksrc[c];
}

}  // namespace dsa
