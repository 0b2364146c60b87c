// Top-k token selector (stage 2): per query row, the topk keys with the largest indexer score
// among keys 0..pos(t); equal scores go to the smaller key index; rows with fewer than topk
// prior keys keep all of them.  ("top-k=2048", "DeepSeek V3.2-Exp Cuts Long-Context Costs with
// DeepSeek Sparse Attention (DSA)", "Training signal"; "Top-k Token Selection", maplevalley
// page, section 1.)
//
// Radix select, no sort: each score maps to a 32-bit key whose unsigned order is the float
// order (-0 folded onto +0).  Three histogram passes over the row (digits of 11, 11 and 10
// bits, most significant first, each restricted to the keys that match the digits fixed so
// far) pin the exact k-th key tau and how many keys equal to tau are still needed.  A final
// pass walks the row in index order with block-wide scans: every key > tau is taken, and the
// first `need` keys == tau (the smallest indices) are taken.  Output: the selected indices in
// increasing order, then -1 padding.  One CTA of 1024 threads per row; rows are read with
// 16-byte vector loads (the score slab stays in L2 between the indexer and this kernel).
#pragma once
#include "sm100.cuh"

namespace dsa {

struct TopkParams {
  const float* scores;     // slab row 0
  int64_t ld;
  int32_t* idx;            // [row_count, topk]
  int32_t topk;
  int32_t decode;
  int32_t row_begin;
  int32_t batch;
  const int32_t* cu_seqlens;
  const int32_t* seq_lens;
  int32_t max_seqlen;
  int32_t* status;
};

constexpr int kTopkThreads = 1024;

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0) u = 0;                       // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block scan of one value per thread; returns the prefix, *total gets the sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_tmp,
                                                    uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_tmp[lane];
    uint32_t t = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_tmp[lane] = t - w;                       // exclusive prefix of warp sums
    if (lane == 31) warp_tmp[32] = t;
  }
  __syncthreads();
  const uint32_t res = warp_tmp[warp] + x - v;
  *total = warp_tmp[32];
  __syncthreads();                                // warp_tmp reusable afterwards
  return res;
}

__global__ void __launch_bounds__(kTopkThreads, 1) dsa_topk_kernel(const TopkParams p) {
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t warp_tmp[33];
  __shared__ uint32_t s_bin, s_above;
  const int tid = threadIdx.x;
  const int r = blockIdx.x;
  const int row = p.row_begin + r;
  int n;
  if (p.decode) {
    n = p.seq_lens[row];
    if (n > p.max_seqlen || n > p.ld) {     // caller error: clamp to the slab and report
      if (tid == 0 && p.status) atomicOr(p.status, kStatusBadIndex);
      n = static_cast<int>(min(static_cast<int64_t>(min(n, p.max_seqlen)), p.ld));
    }
  } else {
    int lo = 0, hi = p.batch;                     // largest b with cu[b] <= row
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (p.cu_seqlens[mid] <= row) lo = mid; else hi = mid;
    }
    n = row - p.cu_seqlens[lo] + 1;
  }
  const float* srow = p.scores + static_cast<int64_t>(r) * p.ld;
  int32_t* out = p.idx + static_cast<int64_t>(r) * p.topk;
  const int K = p.topk;
  if (n <= K) {
    for (int j = tid; j < K; j += kTopkThreads) out[j] = j < n ? j : -1;
    return;
  }
  const int n4 = (n + 3) / 4;
  const float4* srow4 = reinterpret_cast<const float4*>(srow);

  uint32_t prefix = 0, mask = 0, need = K;
  constexpr int kShift[3] = {21, 10, 0};
  constexpr int kBits[3] = {11, 11, 10};
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = kShift[pass];
    const uint32_t nb = 1u << kBits[pass];
    for (uint32_t i = tid; i < nb; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    for (int i4 = tid; i4 < n4; i4 += kTopkThreads) {
      const float4 v = srow4[i4];
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (i4 * 4 + e < n) {
          const uint32_t key = score_key(vv[e]);
          if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
        }
      }
    }
    __syncthreads();
    // Descending cumulative count: thread t owns bins in descending order.
    const uint32_t per = nb / kTopkThreads;       // 2 or 1 bins per thread
    uint32_t mine = 0;
    for (uint32_t j = 0; j < per; ++j) mine += hist[nb - 1 - (tid * per + j)];
    uint32_t tot;
    const uint32_t before = block_excl_scan(mine, warp_tmp, &tot);
    if (before < need && before + mine >= need) {
      uint32_t c = before;
      for (uint32_t j = 0; j < per; ++j) {
        const uint32_t bin = nb - 1 - (tid * per + j);
        if (c + hist[bin] >= need) {
          s_bin = bin;
          s_above = c;
          break;
        }
        c += hist[bin];
      }
    }
    __syncthreads();
    const uint32_t bin = s_bin;
    need -= s_above;
    prefix |= bin << shift;
    mask |= (nb - 1) << shift;
    const bool exact = hist[bin] == need;         // every key of this bucket is taken
    __syncthreads();
    if (exact) break;
  }

  // Ordered pass: keys > prefix (under mask) are taken; keys == prefix are taken while the
  // running count of such keys (in index order) is below `need`.
  uint32_t eq_seen = 0, out_pos = 0;
  const int chunk = kTopkThreads * 4;
#pragma unroll 1
  for (int base = 0; base < n; base += chunk) {
    const int i0 = base + tid * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i0 < n) v = srow4[i0 / 4];
    const float vv[4] = {v.x, v.y, v.z, v.w};
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (i0 + e < n) {
        const uint32_t km = score_key(vv[e]) & mask;
        gt |= (km > prefix ? 1u : 0u) << e;
        eq |= (km == prefix ? 1u : 0u) << e;
      }
    }
    uint32_t eq_total;
    const uint32_t eq_before = eq_seen + block_excl_scan(__popc(eq), warp_tmp, &eq_total);
    uint32_t take = gt;
    uint32_t e_rank = eq_before;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if ((eq >> e) & 1u) {
        if (e_rank < need) take |= 1u << e;
        ++e_rank;
      }
    }
    uint32_t take_total;
    uint32_t pos = out_pos + block_excl_scan(__popc(take), warp_tmp, &take_total);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if ((take >> e) & 1u) {
        if (pos < static_cast<uint32_t>(K)) out[pos] = i0 + e;
        ++pos;
      }
    eq_seen += eq_total;
    out_pos += take_total;
  }
  for (int j = out_pos + tid; j < K; j += kTopkThreads) out[j] = -1;
}

}  // namespace dsa
