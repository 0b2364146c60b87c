// Top-k token selector (stage 2): per query row, the topk keys with the largest indexer score
// among keys 0..pos(t); equal scores go to the smaller key index; rows with fewer than topk
// prior keys keep all of them.  ("top-k=2048", "DeepSeek V3.2-Exp Cuts Long-Context Costs with
// DeepSeek Sparse Attention (DSA)", "Training signal"; "Top-k Token Selection", maplevalley
// page, section 1.)
//
// Radix select, no sort.  Each score maps to a 32-bit key whose unsigned order is the float
// order (-0 folded onto +0).  A row is split over a cluster of C CTAs (C = 1..8), CTA c owning
// the slice [c per, (c+1) per) of the row.
//   1. First digit (the top 11 bits of the key).  Its per-row histogram either comes with the
//      scores (the indexer counts each score as it writes it) or is built here with one pass
//      over the slice and summed over the cluster through distributed shared memory.  Every CTA
//      finds the bin b holding the k-th largest key and the count above it.
//   2. One classifying pass over the slice: keys of a bin above b are taken (a bit in the
//      slice's "taken" bitmap); keys of bin b are candidates, kept in shared memory with their
//      positions, each warp in its own region (no shared counter).  When bin b holds exactly
//      the keys still needed, all of it is taken instead.
//      Bitmap layout: a block of 128 keys is 4 words; key 4 l + e of the block is bit l of word
//      e, so that lane l of a warp reading the block as float4 contributes bit l of each word.
//   3. The candidates of the cluster are few (1-6k): their keys go to CTA 0, which resolves the
//      remaining 21 bits (digits of 11 and 10 bits) and broadcasts the exact k-th key tau and the
//      number of keys equal to tau still needed.  Each CTA marks its candidates above tau as
//      taken and those equal to tau as ties (a second bitmap).  A bin too crowded for the
//      buffers (mass ties) is resolved instead with filtered passes over the slice and
//      cluster-summed histograms, followed by a marking pass.
//   4. Output from the bitmaps alone: every taken key, and the first `need` ties in index order
//      (the smaller indices), at positions given by exclusive scans of the per-word counts over
//      the CTA and the cluster, so the indices come out in increasing order.
// The scores are read from global memory once (twice without a given histogram, three times in
// the crowded case), never held in shared memory.
#pragma once
#include "sm100.cuh"

namespace dsa {

struct TopkParams {
  const float* scores;     // slab row 0
  int64_t ld;
  int32_t* idx;            // [row_count, topk]
  float* sel;              // optional [row_count, topk]: the score of each selected key
  int32_t topk;
  int32_t decode;
  int32_t row_begin;
  int32_t batch;
  const int32_t* cu_seqlens;
  const int32_t* seq_lens;
  int32_t max_seqlen;
  int32_t* status;
  int32_t csize;           // CTAs per row (the cluster size)
  int32_t slice;           // keys per CTA slice (a multiple of 128), sizes the bitmaps
  uint32_t* hist;          // optional [row_count][kTopkBins] first-digit counts of each row's
                           // scores; read, then zeroed for the next use
};

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkBins = 2048;
constexpr int kTopkLocal = 4096;     // candidates (key, position) a CTA keeps
constexpr int kTopkPerWarp = kTopkLocal / kTopkWarps;   // each warp's own candidate region
constexpr int kTopkGather = 12288;   // candidate keys CTA 0 gathers from the cluster
constexpr int kTopkFixedSmem =
    2 * kTopkBins * 4 + 2 * kTopkLocal * 4 + kTopkGather * 4 + 512;

// Dynamic shared memory of a launch whose slices hold `slice` keys: the fixed part plus the two
// bitmaps of the slice.
__host__ __device__ constexpr int topk_smem_bytes(int slice) {
  return kTopkFixedSmem + 2 * ((slice + 31) / 32) * 4;
}

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0) u = 0;                       // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The smallest float whose order key is >= t (t <= 2^32): scores compare against it as floats
// exactly as their keys compare against t.  NaN (no float reaches it) for t = 2^32 or inside the
// NaN range of positive keys; -inf when only NaN patterns lie below t (negative keys).
__device__ __forceinline__ float key_floor_float(uint64_t t) {
  if (t >= (uint64_t(1) << 32)) return __int_as_float(0x7fffffff);
  const uint32_t k = static_cast<uint32_t>(t);
  if (k & 0x80000000u) return __uint_as_float(k & 0x7fffffffu);
  const float f = __uint_as_float(~k);
  return f != f ? -INFINITY : f;
}

// Bitmap position of key i of a slice (see the layout above).
__device__ __forceinline__ int bm_word(int i) { return (i >> 7) * 4 + (i & 3); }
__device__ __forceinline__ uint32_t bm_bit(int i) { return 1u << ((i >> 2) & 31); }

__device__ __forceinline__ void st_cluster_u4(uint32_t addr, uint4 v) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void red_cluster_add(uint32_t addr, uint32_t v) {
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Exclusive scan over the CTA's threads (one value each); *total receives the sum.  With
// kReuse the scratch may be used again right after the call (a third barrier); without it the
// caller passes another barrier before tmp is written again.
template <bool kReuse = true>
__device__ __forceinline__ uint32_t cta_excl_scan(uint32_t v, uint32_t* tmp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = lane < kTopkWarps ? tmp[lane] : 0u;
    uint32_t t = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < kTopkWarps) tmp[lane] = t - w;
    if (lane == 31) tmp[32] = t;
  }
  __syncthreads();
  const uint32_t res = tmp[warp] + x - v;
  *total = tmp[32];
  if (kReuse) __syncthreads();
  return res;
}

// Sums the cluster's histograms (nb bins) into every CTA's hsum, which the caller zeroed before
// the histogram was built: every CTA adds its non-zero bins into every CTA's hsum.
__device__ __forceinline__ void cluster_hist_sum(uint32_t* hist, uint32_t* hsum, uint32_t nb,
                                                 int C) {
  if (C > 1) {
    cluster_sync();   // every hist complete, every hsum zeroed
    for (uint32_t i = threadIdx.x; i < nb; i += kTopkThreads) {
      const uint32_t v = hist[i];
      if (v != 0)
        for (int c = 0; c < C; ++c) red_cluster_add(map_to_rank(smem_u32(hsum + i), c), v);
    }
    cluster_sync();
  } else {
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < nb; i += kTopkThreads) hsum[i] = hist[i];
    __syncthreads();
  }
}

// Bin holding the need-th largest key of a histogram of BPT x kTopkThreads bins held in the
// CTA's registers, thread t holding bins [BPT t, BPT t + BPT) in v; every thread gets the same
// (bin, keys in the bins above it, keys in it).  need >= 1.  A histogram holding fewer than
// `need` keys (inconsistent input) gives bin 0 with nothing above it.  Two barriers; the
// scratch (wtot: kTopkWarps words, res: 3) may be written again by the next call at once: its
// reads all precede the second barrier, and the next call writes res only after its first.
template <int BPT>
__device__ __forceinline__ void find_bin(const uint32_t (&v)[BPT], uint32_t need, uint32_t* wtot,
                                         uint32_t* res, uint32_t* bin, uint32_t* above,
                                         uint32_t* in_bin) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t mine = 0;
#pragma unroll
  for (int j = 0; j < BPT; ++j) mine += v[j];
  uint32_t x = mine;                              // this lane's and the higher lanes' keys
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
    if (lane + o < 32) x += y;
  }
  if (lane == 0) wtot[warp] = x;
  __syncthreads();
  uint32_t before = x - mine;                     // keys in the bins above this thread's
  for (int w = warp + 1; w < kTopkWarps; ++w) before += wtot[w];
  if (before < need && before + mine >= need) {   // exactly one thread holds the crossing
    uint32_t c = before;
    bool found = false;
#pragma unroll
    for (int j = BPT - 1; j >= 0; --j) {
      if (!found && c + v[j] >= need) {
        res[0] = static_cast<uint32_t>(BPT * tid + j);
        res[1] = c;
        res[2] = v[j];
        found = true;
      }
      c += v[j];
    }
  } else if (tid == 0 && before + mine < need) {  // fewer keys than needed in all
    res[0] = 0;
    res[1] = 0;
    res[2] = v[0];
  }
  __syncthreads();
  *bin = res[0];
  *above = res[1];
  *in_bin = res[2];
}

// A histogram in shared memory into the registers find_bin takes.
template <int BPT>
__device__ __forceinline__ void load_bins(const uint32_t* h, uint32_t (&v)[BPT]) {
  static_assert(BPT == 2 || BPT == 4, "2 or 4 bins a thread");
  if constexpr (BPT == 4) {
    const uint4 x = reinterpret_cast<const uint4*>(h)[threadIdx.x];
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else {
    const uint2 x = reinterpret_cast<const uint2*>(h)[threadIdx.x];
    v[0] = x.x; v[1] = x.y;
  }
}

__device__ __forceinline__ void cta_or_cluster_sync(int C) {
  if (C > 1) cluster_sync(); else __syncthreads();
}

// two CTAs per SM (64 registers a thread): a row's slices fill one wave in decode
__global__ void __launch_bounds__(kTopkThreads, 2) dsa_topk_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t topk_smem[];
  uint32_t* hsum = reinterpret_cast<uint32_t*>(topk_smem);          // [kTopkBins] row / digit
  uint32_t* hloc = hsum + kTopkBins;                                 // [kTopkBins] this slice
  uint32_t* ckey = hloc + kTopkBins;                                 // [kTopkLocal] candidates
  int32_t* cpos = reinterpret_cast<int32_t*>(ckey + kTopkLocal);     // [kTopkLocal] positions
  uint32_t* gath = reinterpret_cast<uint32_t*>(cpos + kTopkLocal);   // [kTopkGather] (CTA 0)
  uint32_t* tmp = gath + kTopkGather;                                // [40] scan scratch
  uint32_t* cnt = tmp + 40;                                          // [4][8] per-CTA counts
  uint32_t* bc = cnt + 32;                                           // [4] broadcast result
  uint32_t* bm_take = reinterpret_cast<uint32_t*>(topk_smem + kTopkFixedSmem);  // [words]
  const int words = (p.slice + 31) / 32;
  uint32_t* bm_tie = bm_take + words;                                // [words]
  uint32_t* fres = tmp + 36;                                         // [3] find_bin's result
  __shared__ uint32_t s_over;
  __shared__ uint32_t s_wcnt[kTopkWarps];          // candidates of each warp (its region)

  wait_prior_grid();   // (launched early: the scores come from the previous kernel)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = p.csize;
  const int crank = static_cast<int>(blockIdx.x) % C;
  const int r = blockIdx.x / C;
  const int row = p.row_begin + r;
  uint32_t* grow_hist = p.hist ? p.hist + static_cast<int64_t>(r) * kTopkBins : nullptr;
  // the row's first-digit counts are loaded before anything else (their latency then overlaps
  // the row geometry's); thread t holds bins 4t..4t+3
  constexpr int kHpt = kTopkBins / kTopkThreads;
  static_assert(kHpt == 4, "four first-digit bins a thread");
  uint32_t hreg[kHpt];
  if (grow_hist != nullptr) {
    const uint4 h4 = __ldcg(reinterpret_cast<const uint4*>(grow_hist) + tid);
    hreg[0] = h4.x;
    hreg[1] = h4.y;
    hreg[2] = h4.z;
    hreg[3] = h4.w;
  }
  int n;
  if (p.decode) {
    n = p.seq_lens[row];
    if (n > p.max_seqlen || n > p.ld) {     // caller error: clamp to the slab and report
      if (tid == 0 && crank == 0 && p.status) atomicOr(p.status, kStatusBadIndex);
      n = static_cast<int>(min(static_cast<int64_t>(min(n, p.max_seqlen)), p.ld));
    }
  } else {
    int lo = 0, hi = p.batch;                     // largest b with cu[b] <= row
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.cu_seqlens[mid] <= row) lo = mid; else hi = mid;
    }
    n = row - p.cu_seqlens[lo] + 1;
  }
  const float* srow = p.scores + static_cast<int64_t>(r) * p.ld;
  int32_t* out = p.idx + static_cast<int64_t>(r) * p.topk;
  float* sel = p.sel != nullptr ? p.sel + static_cast<int64_t>(r) * p.topk : nullptr;
  const int K = p.topk;
  if (n <= K) {                                    // uniform over the cluster: no barrier used
    for (int j = crank * kTopkThreads + tid; j < K; j += C * kTopkThreads) {
      out[j] = j < n ? j : -1;
      if (sel != nullptr) sel[j] = j < n ? srow[j] : 0.f;
    }
    if (grow_hist != nullptr && crank == 0)        // leave the histogram zeroed for reuse
      for (int i = tid; i < kTopkBins; i += kTopkThreads) grow_hist[i] = 0;
    return;
  }
  // this CTA's slice [s0, s0 + m); per is a multiple of 128 (no larger than p.slice)
  const int per = ((n + C - 1) / C + 127) / 128 * 128;
  const int s0 = min(n, crank * per);
  const int m = min(n, s0 + per) - s0;
  const int nrounds = (m + 127) / 128;           // 128-key blocks: lane l reads keys 4l..4l+3

  for (int i = tid; i < words; i += kTopkThreads) {
    bm_take[i] = 0;
    bm_tie[i] = 0;
  }
  if (tid == 0) s_over = 0;

  // ---- 1. first digit
  if (grow_hist == nullptr) {
    for (int i = tid; i < kTopkBins; i += kTopkThreads) {
      hloc[i] = 0;
      hsum[i] = 0;
    }
    __syncthreads();
    for (int rd = warp; rd < nrounds; rd += kTopkWarps) {
      const int i4 = rd * 128 + 4 * lane;
      if (i4 < m) {
        const float4 v = *reinterpret_cast<const float4*>(srow + s0 + i4);
        atomicAdd(&hloc[score_key(v.x) >> 21], 1u);
        if (i4 + 1 < m) atomicAdd(&hloc[score_key(v.y) >> 21], 1u);
        if (i4 + 2 < m) atomicAdd(&hloc[score_key(v.z) >> 21], 1u);
        if (i4 + 3 < m) atomicAdd(&hloc[score_key(v.w) >> 21], 1u);
      }
    }
    cluster_hist_sum(hloc, hsum, kTopkBins, C);
    load_bins(hsum, hreg);
  }
  uint32_t bin, above, in_bin;
  find_bin(hreg, K, tmp, fres, &bin, &above, &in_bin);
  uint32_t need = K - above;
  const bool whole_bin = in_bin == need;         // every key of the bin is taken
  if (crank == 0 && !whole_bin) {
    // CTA 0's histograms of the second (hloc, 2048 bins) and third (hsum, 1024 bins) digits,
    // zeroed now: the barriers up to the resolution order these stores before its counts
    for (int i = tid; i < kTopkBins; i += kTopkThreads) hloc[i] = 0;
    for (int i = tid; i < kTopkBins / 2; i += kTopkThreads) hsum[i] = 0;
  }
  uint32_t prefix = bin << 21, mask = 0xFFE00000u;

  // ---- 2. classify the slice: above the bin -> taken; in the bin -> candidate
  // (take: key >= t_hi, candidate: t_lo <= key < t_hi; compared as floats, the keys' order,
  // through the smallest float of each threshold's bin)
  const uint32_t t_lo = bin << 21;
  const uint64_t t_hi = whole_bin ? uint64_t(bin) << 21 : (uint64_t(bin) + 1) << 21;
  const float f_lo = key_floor_float(t_lo), f_hi = key_floor_float(t_hi);
  uint32_t* wkey = ckey + warp * kTopkPerWarp;
  int32_t* wpos = cpos + warp * kTopkPerWarp;
  uint32_t wn = 0;                                 // this warp's candidates so far
  constexpr int U = 4;                             // blocks in flight per warp
  for (int rd0 = warp; rd0 < nrounds; rd0 += U * kTopkWarps) {
    float4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i4 = (rd0 + u * kTopkWarps) * 128 + 4 * lane;
      v[u] = i4 < m ? __ldcs(reinterpret_cast<const float4*>(srow + s0 + i4))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int rd = rd0 + u * kTopkWarps;
      if (rd >= nrounds) break;
      const float ve[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint32_t cw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = rd * 128 + 4 * lane + e;
        const bool in = i < m;
        const bool above = ve[e] >= f_hi;
        const uint32_t tw = __ballot_sync(0xffffffffu, in && above);
        if (lane == e) bm_take[rd * 4 + e] = tw;
        cw[e] = __ballot_sync(0xffffffffu, in && !above && ve[e] >= f_lo);
      }
      if ((cw[0] | cw[1] | cw[2] | cw[3]) != 0) {
        // this lane's candidates, in key order (lane-major, then e), into the warp's region
        uint32_t before = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) before += __popc(cw[e] & ((1u << lane) - 1u));
        uint32_t slot = wn + before;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if ((cw[e] >> lane) & 1u) {
            if (slot < static_cast<uint32_t>(kTopkPerWarp)) {
              wkey[slot] = score_key(ve[e]);
              wpos[slot] = rd * 128 + 4 * lane + e;
            }
            ++slot;
          }
        wn += __popc(cw[0]) + __popc(cw[1]) + __popc(cw[2]) + __popc(cw[3]);
      }
    }
  }
  if (lane == 0) {
    s_wcnt[warp] = min(wn, static_cast<uint32_t>(kTopkPerWarp));
    if (wn > static_cast<uint32_t>(kTopkPerWarp)) s_over = 1;
  }
  __syncthreads();

  // ---- 3. resolve tau within the bin
  if (!whole_bin) {
    // each warp's segment padded to a multiple of 4 with a key outside the bin
    const uint32_t pad_key = bin == 0 ? 0xFFFFFFFFu : 0u;
    uint32_t n4 = 0;
    for (int w = 0; w < kTopkWarps; ++w) n4 += (s_wcnt[w] + 3u) & ~3u;
    // every CTA learns every CTA's candidate count and overflow flag
    if (tid == 0) {
      for (int c = 0; c < C; ++c) {
        const uint32_t a = C > 1 ? map_to_rank(smem_u32(cnt), c) : smem_u32(cnt);
        if (C > 1) {
          st_cluster_u32(a + 4 * crank, n4);
          st_cluster_u32(a + 4 * (8 + crank), s_over);
        } else {
          cnt[0] = n4;
          cnt[8] = s_over;
        }
      }
    }
    cta_or_cluster_sync(C);
    uint32_t total = 0, off = 0, over = 0;
    for (int c = 0; c < C; ++c) {
      if (c < crank) off += cnt[c];
      total += cnt[c];
      over |= cnt[8 + c];
    }
    const bool crowded = over != 0 || total > static_cast<uint32_t>(kTopkGather);
    if (!crowded) {
      // candidates' keys into CTA 0, each warp its own padded segment, 16 B at a time
      {
        uint32_t woff = off;                       // this warp's segment in CTA 0's buffer
        for (int w = 0; w < warp; ++w) woff += (s_wcnt[w] + 3u) & ~3u;
        const uint32_t wc = s_wcnt[warp], w4 = (wc + 3u) & ~3u;
        if (lane < static_cast<int>(w4 - wc)) wkey[wc + lane] = pad_key;
        __syncwarp();
        const uint4* src4 = reinterpret_cast<const uint4*>(wkey);
        if (C > 1) {
          const uint32_t dst0 = map_to_rank(smem_u32(gath), 0) + woff * 4;
          for (uint32_t j = lane; j < w4 / 4; j += 32) st_cluster_u4(dst0 + j * 16, src4[j]);
        } else {
          for (uint32_t j = lane; j < w4 / 4; j += 32)
            reinterpret_cast<uint4*>(gath + woff)[j] = src4[j];
        }
      }
      cta_or_cluster_sync(C);                      // CTA 0 holds every candidate
      if (crank == 0) {
        // second digit (11 bits) into hloc, then, unless its bin is exact, the third (10 bits)
        // into hsum; both were zeroed before the classifying pass
        for (uint32_t i = tid; i < total; i += kTopkThreads) {
          const uint32_t k = gath[i];
          if ((k & mask) == prefix) atomicAdd(&hloc[(k >> 10) & 2047u], 1u);
        }
        __syncthreads();
        uint32_t v2[4], b2, ab2, nb2;
        load_bins(hloc, v2);
        find_bin(v2, need, tmp, fres, &b2, &ab2, &nb2);
        need -= ab2;
        prefix |= b2 << 10;
        mask |= 2047u << 10;
        if (nb2 != need) {
          for (uint32_t i = tid; i < total; i += kTopkThreads) {
            const uint32_t k = gath[i];
            if ((k & mask) == prefix) atomicAdd(&hsum[k & 1023u], 1u);
          }
          __syncthreads();
          uint32_t v3[2], b3, ab3, nb3;
          load_bins(hsum, v3);
          find_bin(v3, need, tmp, fres, &b3, &ab3, &nb3);
          need -= ab3;
          prefix |= b3;
          mask |= 1023u;
        }
        if (tid == 0)
          for (int c = 0; c < C; ++c) {
            if (C > 1) {
              const uint32_t a = map_to_rank(smem_u32(bc), c);
              st_cluster_u32(a + 0, prefix);
              st_cluster_u32(a + 4, mask);
              st_cluster_u32(a + 8, need);
            } else {
              bc[0] = prefix;
              bc[1] = mask;
              bc[2] = need;
            }
          }
      }
      cta_or_cluster_sync(C);                      // the broadcast has landed
      prefix = bc[0];
      mask = bc[1];
      need = bc[2];
      // mark the candidates: above tau -> taken, equal -> tie
      for (uint32_t j = lane; j < s_wcnt[warp]; j += 32) {
        const uint32_t km = wkey[j] & mask;
        const int i = wpos[j];
        if (km > prefix) atomicOr(&bm_take[bm_word(i)], bm_bit(i));
        else if (km == prefix) atomicOr(&bm_tie[bm_word(i)], bm_bit(i));
      }
    } else {
      // crowded bin: the remaining digits with filtered passes and cluster sums, then a pass
      // that marks the bin's keys
      constexpr int kShift[2] = {10, 0};
      constexpr int kBits[2] = {11, 10};
      for (int pass = 0; pass < 2; ++pass) {
        const uint32_t nb = 1u << kBits[pass];
        for (uint32_t i = tid; i < nb; i += kTopkThreads) {
          hloc[i] = 0;
          hsum[i] = 0;
        }
        __syncthreads();
        for (int i = tid; i < m; i += kTopkThreads) {
          const uint32_t k = score_key(srow[s0 + i]);
          if ((k & mask) == prefix) atomicAdd(&hloc[(k >> kShift[pass]) & (nb - 1)], 1u);
        }
        cluster_hist_sum(hloc, hsum, nb, C);
        uint32_t b2, ab2, nb2;
        if (pass == 0) {
          uint32_t v2[4];
          load_bins(hsum, v2);
          find_bin(v2, need, tmp, fres, &b2, &ab2, &nb2);
        } else {
          uint32_t v3[2];
          load_bins(hsum, v3);
          find_bin(v3, need, tmp, fres, &b2, &ab2, &nb2);
        }
        need -= ab2;
        prefix |= b2 << kShift[pass];
        mask |= (nb - 1) << kShift[pass];
        if (nb2 == need) break;
      }
      for (int i = tid; i < m; i += kTopkThreads) {
        const uint32_t k = score_key(srow[s0 + i]);
        if ((k >> 21) != bin) continue;            // the bin's keys only (above: taken already)
        const uint32_t km = k & mask;
        if (km > prefix) atomicOr(&bm_take[bm_word(i)], bm_bit(i));
        else if (km == prefix) atomicOr(&bm_tie[bm_word(i)], bm_bit(i));
      }
    }
  }
  __syncthreads();

  // ---- 4. output: taken keys and the first `need` ties, in index order
  // thread t owns the 128-key blocks [t bpt, (t+1) bpt) of the slice
  const int nblk = words / 4;
  const int bpt = (nblk + kTopkThreads - 1) / kTopkThreads;
  const int b0 = min(nblk, tid * bpt), b1 = min(nblk, b0 + bpt);
  uint32_t tk = 0, te = 0;
  for (int w = 4 * b0; w < 4 * b1; ++w) {
    tk += __popc(bm_take[w]);
    te += __popc(bm_tie[w]);
  }
  // one scan of both counts packed in 16-bit halves when a slice cannot hold 65536 keys of a
  // kind (taken keys are at most topk), else two scans
  uint32_t tk_before, te_before, tk_tot, te_tot;
  if (m < 65536) {
    uint32_t both_tot;   // (tmp is not written again before the next barrier)
    const uint32_t both_before = cta_excl_scan<false>(tk | (te << 16), tmp, &both_tot);
    tk_before = both_before & 0xffffu;
    te_before = both_before >> 16;
    tk_tot = both_tot & 0xffffu;
    te_tot = both_tot >> 16;
  } else {
    tk_before = cta_excl_scan(tk, tmp, &tk_tot);
    te_before = cta_excl_scan<false>(te, tmp, &te_tot);
  }
  if (tid == 0) {
    for (int c = 0; c < C; ++c) {
      if (C > 1) {
        const uint32_t a = map_to_rank(smem_u32(cnt), c);
        st_cluster_u32(a + 4 * (16 + crank), tk_tot);
        st_cluster_u32(a + 4 * (24 + crank), te_tot);
      } else {
        cnt[16] = tk_tot;
        cnt[24] = te_tot;
      }
    }
  }
  cta_or_cluster_sync(C);
  uint32_t tk0 = 0, te0 = 0;                       // the CTAs before this one
  for (int c = 0; c < crank; ++c) {
    tk0 += cnt[16 + c];
    te0 += cnt[24 + c];
  }
  tk_before += tk0;
  te_before += te0;
  if (grow_hist != nullptr && crank == 0)         // every CTA has read it: zero for reuse
    for (int i = tid; i < kTopkBins; i += kTopkThreads) grow_hist[i] = 0;
  for (int blk = b0; blk < b1; ++blk) {
    uint32_t t[4], e[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      t[q] = bm_take[4 * blk + q];
      e[q] = bm_tie[4 * blk + q];
    }
    uint32_t any = (t[0] | e[0]) | (t[1] | e[1]) | (t[2] | e[2]) | (t[3] | e[3]);
    while (any) {                                  // key 4 l + q of the block, l ascending
      const int l = __ffs(any) - 1;
      any &= any - 1;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t pos = 0xFFFFFFFFu;
        if ((t[q] >> l) & 1u) {
          pos = tk_before + min(te_before, need);
          ++tk_before;
        } else if ((e[q] >> l) & 1u) {
          if (te_before < need) pos = tk_before + te_before;
          ++te_before;
        }
        if (pos < static_cast<uint32_t>(K)) out[pos] = s0 + blk * 128 + 4 * l + q;
      }
    }
  }
  if (sel != nullptr) {
    // the slice's outputs are one contiguous range of positions (keys in increasing order):
    // every thread fetches scores of it, all loads in flight together
    const uint32_t ties = need > te0 ? min(need - te0, te_tot) : 0u;
    const uint32_t begin = tk0 + min(te0, need), count = tk_tot + ties;
    __syncthreads();                               // this CTA's indices are written
    for (uint32_t j = begin + tid; j < begin + count && j < static_cast<uint32_t>(K);
         j += kTopkThreads)
      sel[j] = srow[out[j]];
  }
  // no CTA may leave while a peer can still write into its shared memory: the last remote
  // writes were the counts above, ordered before the barrier that every CTA has passed
}

}  // namespace dsa
