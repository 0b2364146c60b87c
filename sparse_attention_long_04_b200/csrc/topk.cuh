// Top-k token selector (stage 2): per query row, the topk keys with the largest indexer score
// among keys 0..pos(t); equal scores go to the smaller key index; rows with fewer than topk
// prior keys keep all of them.  ("top-k=2048", "DeepSeek V3.2-Exp Cuts Long-Context Costs with
// DeepSeek Sparse Attention (DSA)", "Training signal"; "Top-k Token Selection", maplevalley
// page, section 1.)
//
// Radix select, no sort.  Each score maps to a 32-bit key whose unsigned order is the float
// order (-0 folded onto +0).  A row is split over a cluster of C CTAs (C = 1..8); CTA c reads
// its slice of the row from global memory once and keeps the keys in shared memory, building
// the histogram of the first digit (the top 11 bits) while it loads.  The C histograms are
// summed through distributed shared memory (each CTA adds its non-zero bins into every CTA)
// and every CTA picks the bin holding the k-th largest key.  The keys of that bin are few:
// every CTA appends its own into CTA 0's candidate buffer, CTA 0 resolves the remaining 21
// bits (digits of 11 and 10 bits) locally and broadcasts the exact k-th key tau and the count
// of keys == tau still needed.  (If the bin is too crowded for the buffer, e.g. mass ties, the
// CTAs resolve the remaining digits together with filtered scans and cluster-summed
// histograms instead.)  The output pass takes every key > tau and the first `need` keys == tau in index
// order (the smallest indices): per-warp counts give each warp's output offset (an exclusive
// scan over the cluster in index order), and the indices come out in increasing order.
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
  int32_t csize;           // CTAs per row (the cluster size)
};

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkSlice = 16384;          // keys a CTA keeps in shared memory
constexpr int kTopkBins = 2048;
constexpr int kTopkCand = 8192;           // candidate keys CTA 0 gathers after the first digit
// 112.5 KiB: two CTAs still fit on one SM
constexpr int kTopkSmem = kTopkSlice * 4 + kTopkCand * 4 + 2 * kTopkBins * 4 + 512;

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0) u = 0;                       // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint4 ld_cluster_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_cluster_u4(uint32_t addr, uint4 v) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Exclusive scan over the CTA's threads (one value each); *total receives the sum.
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
  __syncthreads();
  return res;
}

__device__ __forceinline__ void red_cluster_add(uint32_t addr, uint32_t v) {
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
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

__device__ __forceinline__ uint32_t atom_cluster_add(uint32_t addr, uint32_t v) {
  uint32_t old;
  asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v)
               : "memory");
  return old;
}

// Bin holding the need-th largest key of hsum (nb bins, descending cumulative counts); all
// threads of the CTA call it and all get the same (bin, count above the bin).
__device__ __forceinline__ void find_bin(const uint32_t* hsum, uint32_t nb, uint32_t need,
                                         uint32_t* tmp, uint32_t* s_bin, uint32_t* s_above,
                                         uint32_t* bin, uint32_t* above) {
  const int tid = threadIdx.x;
  const uint32_t bpt = nb / kTopkThreads;         // 4 or 2 bins per thread
  uint32_t mine = 0;
  for (uint32_t j = 0; j < bpt; ++j) mine += hsum[nb - 1 - (tid * bpt + j)];
  uint32_t tot;
  const uint32_t before = cta_excl_scan(mine, tmp, &tot);
  if (before < need && before + mine >= need) {
    uint32_t c = before;
    for (uint32_t j = 0; j < bpt; ++j) {
      const uint32_t b = nb - 1 - (tid * bpt + j);
      if (c + hsum[b] >= need) {
        *s_bin = b;
        *s_above = c;
        break;
      }
      c += hsum[b];
    }
  }
  __syncthreads();
  *bin = *s_bin;
  *above = *s_above;
  __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads) dsa_topk_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t topk_smem[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(topk_smem);           // [kTopkSlice]
  uint32_t* cand = keys + kTopkSlice;                                // [kTopkCand] (CTA 0)
  uint32_t* hist = cand + kTopkCand;                                 // [kTopkBins] this CTA
  uint32_t* hsum = hist + kTopkBins;                                 // [kTopkBins] cluster sum
  uint32_t* tmp = hsum + kTopkBins;                                  // [40] scan scratch
  uint32_t* wgt = tmp + 40;                                          // [16] per-warp > tau
  uint32_t* weq = wgt + 16;                                          // [16] per-warp == tau
  uint32_t* cnt = weq + 16;                                          // [16] per-CTA (gt, eq)
  uint32_t* bc = cnt + 16;                                           // [4] broadcast result
  __shared__ uint32_t s_bin, s_above, s_ncand, s_base;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = p.csize;
  const int crank = static_cast<int>(blockIdx.x) % C;
  const int r = blockIdx.x / C;
  const int row = p.row_begin + r;
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
  const int K = p.topk;
  if (n <= K) {                                    // uniform over the cluster: no barrier used
    for (int j = crank * kTopkThreads + tid; j < K; j += C * kTopkThreads)
      out[j] = j < n ? j : -1;
    return;
  }
  // this CTA's slice [s0, s1); a multiple of 4 long so every slice starts 16-byte aligned
  const int per = ((n + C - 1) / C + 3) / 4 * 4;
  const int s0 = min(n, crank * per);
  const int s1 = min(n, s0 + per);
  const int m = s1 - s0;
  const bool cached = m <= kTopkSlice;
  auto key_at = [&](int i) -> uint32_t {
    return cached ? keys[i] : score_key(srow[s0 + i]);
  };
  auto key4_at = [&](int i) -> uint4 {            // i multiple of 4, i < m
    if (cached) return *reinterpret_cast<const uint4*>(keys + i);
    if (i + 3 < m) {                              // a streamed slice: one 16-byte load
      const float4 v = *reinterpret_cast<const float4*>(srow + s0 + i);
      return make_uint4(score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w));
    }
    uint4 k = make_uint4(0, 0, 0, 0);
    if (i + 0 < m) k.x = score_key(srow[s0 + i + 0]);
    if (i + 1 < m) k.y = score_key(srow[s0 + i + 1]);
    if (i + 2 < m) k.z = score_key(srow[s0 + i + 2]);
    if (i + 3 < m) k.w = score_key(srow[s0 + i + 3]);
    return k;
  };

  // ---- digit 1 (top 11 bits): load + histogram in one pass
  for (int i = tid; i < kTopkBins; i += kTopkThreads) {
    hist[i] = 0;
    hsum[i] = 0;
  }
  if (tid == 0) s_ncand = 0;
  __syncthreads();
  if (cached) {
    constexpr int kVec = kTopkSlice / 4 / kTopkThreads;   // float4 per thread (8)
    float4 v[kVec];
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      const int i4 = (u * kTopkThreads + tid) * 4;
      v[u] = i4 < m ? *reinterpret_cast<const float4*>(srow + s0 + i4)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      const int i4 = (u * kTopkThreads + tid) * 4;
      if (i4 < m) {
        const uint4 k = make_uint4(score_key(v[u].x), score_key(v[u].y), score_key(v[u].z),
                                   score_key(v[u].w));
        *reinterpret_cast<uint4*>(keys + i4) = k;
        atomicAdd(&hist[k.x >> 21], 1u);
        if (i4 + 1 < m) atomicAdd(&hist[k.y >> 21], 1u);
        if (i4 + 2 < m) atomicAdd(&hist[k.z >> 21], 1u);
        if (i4 + 3 < m) atomicAdd(&hist[k.w >> 21], 1u);
      }
    }
  } else {
    // a slice longer than shared memory holds: streamed with 16-byte loads, 4 in flight
    for (int base = tid * 4; base < m; base += kTopkThreads * 16) {
      uint4 k[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i4 = base + u * kTopkThreads * 4;
        k[u] = i4 < m ? key4_at(i4) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i4 = base + u * kTopkThreads * 4;
        if (i4 < m) atomicAdd(&hist[k[u].x >> 21], 1u);
        if (i4 + 1 < m) atomicAdd(&hist[k[u].y >> 21], 1u);
        if (i4 + 2 < m) atomicAdd(&hist[k[u].z >> 21], 1u);
        if (i4 + 3 < m) atomicAdd(&hist[k[u].w >> 21], 1u);
      }
    }
  }
  cluster_hist_sum(hist, hsum, kTopkBins, C);
  uint32_t bin, above;
  find_bin(hsum, kTopkBins, K, tmp, &s_bin, &s_above, &bin, &above);
  uint32_t need = K - above;
  uint32_t prefix = bin << 21, mask = 0xFFE00000u;
  const uint32_t in_bin_total = hsum[bin];
  const uint32_t in_bin_local = hist[bin];
  __syncthreads();

  if (in_bin_total != need) {                     // else: every key of the bin is taken
    if (in_bin_total + 3u * C <= static_cast<uint32_t>(kTopkCand)) {
      // ---- gather the bin's keys into CTA 0 and resolve the last 21 bits there.  Each CTA
      // reserves a multiple of 4 slots, compacts its keys locally (CTA 0: in place), pads with
      // a key outside the bin and copies 16 bytes at a time into CTA 0's buffer.
      const uint32_t n4 = (in_bin_local + 3u) & ~3u;
      const uint32_t pad_key = bin == 0 ? 0xFFFFFFFFu : 0u;   // never matches the bin
      if (tid == 0)
        s_base = n4 ? (C > 1 ? atom_cluster_add(map_to_rank(smem_u32(&s_ncand), 0), n4)
                             : atomicAdd(&s_ncand, n4))
                    : 0u;
      if (C > 1) cluster_sync(); else __syncthreads();   // reservations done (CTA 0's count)
      uint32_t mine = 0;                           // this thread's matches, in its 4-key groups
      const int nrounds = (m + kTopkThreads * 4 - 1) / (kTopkThreads * 4);
      for (int u = 0; u < nrounds; ++u) {
        const int i4 = (u * kTopkThreads + tid) * 4;
        if (i4 < m) {
          const uint4 k = key4_at(i4);
          mine += (k.x & mask) == prefix;
          mine += i4 + 1 < m && (k.y & mask) == prefix;
          mine += i4 + 2 < m && (k.z & mask) == prefix;
          mine += i4 + 3 < m && (k.w & mask) == prefix;
        }
      }
      uint32_t tot;
      const uint32_t lbase = crank == 0 ? s_base : 0u;   // where this CTA compacts locally
      uint32_t slot = lbase + cta_excl_scan(mine, tmp, &tot);
      for (int u = 0; u < nrounds && mine; ++u) {
        const int i4 = (u * kTopkThreads + tid) * 4;
        if (i4 < m) {
          const uint4 k = key4_at(i4);
          const uint32_t kk[4] = {k.x, k.y, k.z, k.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (i4 + e < m && (kk[e] & mask) == prefix) cand[slot++] = kk[e];
        }
      }
      if (tid < static_cast<int>(n4 - in_bin_local)) cand[lbase + in_bin_local + tid] = pad_key;
      __syncthreads();
      if (C > 1 && crank != 0) {
        const uint32_t dst0 = map_to_rank(smem_u32(cand), 0) + s_base * 4;
        const uint4* src4 = reinterpret_cast<const uint4*>(cand);
        for (uint32_t j = tid; j < n4 / 4; j += kTopkThreads) st_cluster_u4(dst0 + j * 16, src4[j]);
      }
      if (C > 1) cluster_sync(); else __syncthreads();   // CTA 0 holds every candidate
      if (crank == 0) {
        // digits 2 and 3 over the candidates, locally
        constexpr int kShift[2] = {10, 0};
        constexpr int kBits[2] = {11, 10};
        for (int pass = 0; pass < 2; ++pass) {
          const uint32_t nb = 1u << kBits[pass];
          for (uint32_t i = tid; i < nb; i += kTopkThreads) hsum[i] = 0;
          __syncthreads();
          for (uint32_t i = tid; i < s_ncand; i += kTopkThreads) {
            const uint32_t k = cand[i];
            if ((k & mask) == prefix) atomicAdd(&hsum[(k >> kShift[pass]) & (nb - 1)], 1u);
          }
          __syncthreads();
          uint32_t b2, ab2;
          find_bin(hsum, nb, need, tmp, &s_bin, &s_above, &b2, &ab2);
          need -= ab2;
          prefix |= b2 << kShift[pass];
          mask |= (nb - 1) << kShift[pass];
          const bool exact = hsum[b2] == need;
          __syncthreads();
          if (exact) break;
        }
        if (tid == 0)
          for (int c = 0; c < C; ++c) {
            const uint32_t base = C > 1 ? map_to_rank(smem_u32(bc), c) : smem_u32(bc);
            if (C > 1) {
              st_cluster_u32(base + 0, prefix);
              st_cluster_u32(base + 4, mask);
              st_cluster_u32(base + 8, need);
            } else {
              bc[0] = prefix;
              bc[1] = mask;
              bc[2] = need;
            }
          }
      }
      if (C > 1) cluster_sync(); else __syncthreads();   // the broadcast has landed
      prefix = bc[0];
      mask = bc[1];
      need = bc[2];
    } else {
      // ---- crowded bin: the remaining digits with filtered scans and cluster sums
      constexpr int kShift[2] = {10, 0};
      constexpr int kBits[2] = {11, 10};
      for (int pass = 0; pass < 2; ++pass) {
        const uint32_t nb = 1u << kBits[pass];
        for (uint32_t i = tid; i < nb; i += kTopkThreads) {
          hist[i] = 0;
          hsum[i] = 0;
        }
        __syncthreads();
        for (int i = tid; i < m; i += kTopkThreads) {
          const uint32_t k = key_at(i);
          if ((k & mask) == prefix) atomicAdd(&hist[(k >> kShift[pass]) & (nb - 1)], 1u);
        }
        cluster_hist_sum(hist, hsum, nb, C);
        uint32_t b2, ab2;
        find_bin(hsum, nb, need, tmp, &s_bin, &s_above, &b2, &ab2);
        need -= ab2;
        prefix |= b2 << kShift[pass];
        mask |= (nb - 1) << kShift[pass];
        const bool exact = hsum[b2] == need;
        __syncthreads();
        if (exact) break;
      }
    }
  }

  // ---- output: keys > tau, then the first `need` keys == tau in index order
  const int wn = ((m + kTopkWarps - 1) / kTopkWarps + 127) / 128 * 128;   // per warp, x128
  const int w0 = min(m, warp * wn), w1 = min(m, w0 + wn);
  uint32_t gt = 0, eq = 0;
  for (int i4 = w0 + lane * 4; i4 < w1; i4 += 128) {
    const uint4 k = key4_at(i4);
    const uint32_t kk[4] = {k.x, k.y, k.z, k.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (i4 + e < w1) {
        const uint32_t km = kk[e] & mask;
        gt += km > prefix;
        eq += km == prefix;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  if (lane == 0) {
    wgt[warp] = gt;
    weq[warp] = eq;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t g = 0, e = 0;
    for (int w = 0; w < kTopkWarps; ++w) {
      g += wgt[w];
      e += weq[w];
    }
    if (C > 1) {
      for (int c = 0; c < C; ++c) {
        st_cluster_u32(map_to_rank(smem_u32(cnt + crank), c), g);
        st_cluster_u32(map_to_rank(smem_u32(cnt + 8 + crank), c), e);
      }
    } else {
      cnt[0] = g;
      cnt[8] = e;
    }
  }
  if (C > 1) cluster_sync(); else __syncthreads();
  // every key == tau is taken when the cluster holds exactly `need` of them (the usual case)
  uint32_t eq_all = 0;
  for (int c = 0; c < C; ++c) eq_all += cnt[8 + c];
  const bool all_eq = eq_all == need;
  // offsets: keys taken by the CTAs, then the warps, before this one (index order)
  uint32_t w_out = 0, w_eq = 0;
  for (int c = 0; c < crank; ++c) {
    w_out += cnt[c] + (need > w_eq ? min(need - w_eq, cnt[8 + c]) : 0u);
    w_eq += cnt[8 + c];
  }
  for (int w = 0; w < warp; ++w) {
    w_out += wgt[w] + (need > w_eq ? min(need - w_eq, weq[w]) : 0u);
    w_eq += weq[w];
  }
  // 128 keys per round: lane j holds keys 4j..4j+3 of the round (index order = lane order).
  // Few keys are taken (topk of the row): a warp with none skips the loop, a round with none
  // skips the scans.
  const bool warp_has = wgt[warp] + weq[warp] != 0;
  for (int b0 = w0; warp_has && b0 < w1; b0 += 128) {
    const int i4 = b0 + lane * 4;
    const uint4 k = i4 < w1 ? key4_at(i4) : make_uint4(0, 0, 0, 0);
    const uint32_t kk[4] = {k.x, k.y, k.z, k.w};
    uint32_t gtm = 0, eqm = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (i4 + e < w1) {
        const uint32_t km = kk[e] & mask;
        gtm |= (km > prefix ? 1u : 0u) << e;
        eqm |= (km == prefix ? 1u : 0u) << e;
      }
    }
    if (!__any_sync(0xffffffffu, (gtm | eqm) != 0)) continue;   // nothing here: offsets unchanged
    // counts over the lanes before this one (index order) from one ballot per key slot
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t take = gtm | eqm;
    uint32_t round_eq = 0;
    if (!all_eq) {
      uint32_t eq_before = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t be = __ballot_sync(0xffffffffu, (eqm >> e) & 1u);
        eq_before += __popc(be & lt);
        round_eq += __popc(be);
      }
      uint32_t eq_rank = w_eq + eq_before;      // rank of this lane's first key == tau
      take = gtm;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if ((eqm >> e) & 1u) {
          if (eq_rank < need) take |= 1u << e;
          ++eq_rank;
        }
    }
    uint32_t before = 0, round_take = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t bt = __ballot_sync(0xffffffffu, (take >> e) & 1u);
      before += __popc(bt & lt);
      round_take += __popc(bt);
    }
    uint32_t pos = w_out + before;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if ((take >> e) & 1u) {
        if (pos < static_cast<uint32_t>(K)) out[pos] = s0 + i4 + e;
        ++pos;
      }
    w_out += round_take;
    if (!all_eq) w_eq += round_eq;
  }
}

}  // namespace dsa
