// Sparse MLA attention in MQA mode (stage 3) and the split-KV combine.
//
// For query row t, head h, over the selected logical keys I_t (idx >= 0):
//   l_s = sigma * q[t,h,:] . kv[s,:]            (all D_QK = latent + RoPE dims)
//   O[t,h,:] = sum_s softmax(l)_s * kv[s, 0:D_V] (values = the first D_V latent dims)
//   LSE[t,h] = log sum_s exp(l_s)
// Every selected latent row serves all query heads: MLA run in its multi-query form
// ("DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek Sparse Attention (DSA)",
// "Instantiation").
//
// Design (sm_100a).  O for 128 heads x 512 values in fp32 is 256 KB = all of one SM's TMEM,
// so each query row runs on two CTAs: CTA v (v = 0, 1) accumulates the value dims
// [v D_V/2, (v+1) D_V/2) and, to need nothing from its partner, computes the full logits of
// every tile itself (the QK product is done twice; the two CTAs exchange no data).  Both run
// the same instructions on the same inputs, so their logits, softmax and LSE agree bit for bit.
//   Q (128 heads x 576 bf16) is the QK A operand: TMA brings it in as 128-byte-swizzled 64-dim
//   blocks; the first KBT blocks move on into Tensor Memory (2 bf16 per column), the rest stay
//   in shared memory.  Every selected key is resolved to its physical cache row once, up front
//   (invalid keys borrow a valid row of their tile and are masked out of the softmax); the rows
//   of each 64-key tile (all dims) are then gathered by TMA, four rows per instruction, into a
//   2-stage ring.  Per tile: S = Q K^T (tcgen05 bf16, M = 128 heads, N = 64 keys, fp32 in
//   TMEM), an online softmax (thread = head = TMEM lane), P (bf16) back into TMEM, and
//   O_v += P V_v (A = P from TMEM, N = D_V/2, V read MN-major straight out of the gathered
//   tile).  Rescaling of O is lazy (only when a tile's max beats the running reference by more
//   than 2^8, so P <= 256).
// TMEM columns: O [0, D_V/2) | S [+64) | P [+32) | Q (KBT x 32 columns).
// Warp roles per CTA (512 threads): warp 0 loads Q and issues QK, warp 2 issues PV, warp 1
// owns TMEM, warps 4-11 move Q into TMEM and run the softmax (warps 4-7 take keys 0-31 of a
// tile, warps 8-11 keys 32-63) and the epilogue, warps 12-15 resolve the keys and gather (warp
// w: rows [16w, 16w + 16) of every tile).  Grid: x = 2 * row + v, y = split-KV slice.
#pragma once
#include "sm100.cuh"

namespace dsa {

struct MlaParams {
  const __nv_bfloat16* q;      // [T, H, D_QK]
  const __nv_bfloat16* kv;     // [R, D_QK]
  const int32_t* idx;          // [row_count, topk], relative to row_begin
  __nv_bfloat16* out;          // [T, H, D_V]
  float* lse;                  // [T, H]
  float* part_o;               // split-KV partials [splits, row_count, H, D_V] or null
  float* part_lse;             // [splits, row_count, H]
  int32_t row_begin, row_count, topk, h, splits;
  float scale_log2;            // sigma * log2(e)
  int32_t decode;
  int32_t batch;
  const int32_t* cu_seqlens;
  const int32_t* seq_lens;
  const int32_t* block_table;
  int32_t max_blocks;
  int32_t kv_stride;
  int32_t max_seqlen;
  int32_t block_size;
  int64_t num_kv_rows;
  int32_t* status;
};

template <int D_QK, int D_V>
struct MlaCfg {
  static constexpr int KB_ALL = (D_QK + 63) / 64;     // 64-element k-blocks of a latent row
  static constexpr int V_HALF = D_V / 2;              // value dims per CTA
  static constexpr int VKB = V_HALF / 64;             // value k-blocks per CTA
  static constexpr int BN = 64;                       // keys per tile
  static constexpr int STAGES = 2;
  static constexpr int MAX_TILES = 32;                // topk <= 2048
  static constexpr int THREADS = 512;
  static constexpr int S_COL = V_HALF;
  static constexpr int P_COL = S_COL + BN;
  static constexpr int Q_COL = P_COL + BN / 2;
  static constexpr int KBT_MAX = (512 - Q_COL) / 32;
  static constexpr int KBT = KB_ALL < KBT_MAX ? KB_ALL : KBT_MAX;   // Q k-blocks in TMEM
  static constexpr int KBS = KB_ALL - KBT;                            // Q k-blocks in smem
  static constexpr int TMEM_COLS = Q_COL + KBT * 32 <= 256 ? 256 : 512;
  static constexpr int KB_BYTES = BN * 128;                           // one k-block of a tile
  static constexpr int KV_STAGE_BYTES = KB_ALL * KB_BYTES;
  static constexpr int Q_KB_BYTES = 128 * 128;                        // one k-block of Q
  static constexpr int Q_SMEM_BYTES = KBS * Q_KB_BYTES;
  static constexpr int ROWS_PER_WARP_TX = 16 * KB_ALL * 128;          // gather bytes per warp
  static constexpr int SMEM_USED = 1024 + Q_SMEM_BYTES + STAGES * KV_STAGE_BYTES +
                                   MAX_TILES * BN * 4 + MAX_TILES * 12 + 2 * 2 * 128 * 4 +
                                   2 * 128 * 4 + 256;
  // at least 116 KB, so that one CTA runs per SM (its TMEM allocation never waits)
  static constexpr int SMEM_BYTES = SMEM_USED > 116 * 1024 ? SMEM_USED : 116 * 1024;
  static_assert(V_HALF % 64 == 0 && V_HALF <= 256, "PV MMA N");
  static_assert(Q_COL + KBT * 32 <= 512, "TMEM columns");
  static_assert(KBT * Q_KB_BYTES <= STAGES * KV_STAGE_BYTES, "Q staging fits the gather ring");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <int D_QK, int D_V>
__global__ void __launch_bounds__(512, 1)
    dsa_sparse_mla_kernel(const __grid_constant__ CUtensorMap kv_map,
                          const __grid_constant__ CUtensorMap q_map, const MlaParams p) {
  using C = MlaCfg<D_QK, D_V>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                                           // [KBS][128 heads][128 B]
  uint8_t* sKV = sQ + C::Q_SMEM_BYTES;                          // [STAGES] gathered tiles
  int32_t* sPhys = reinterpret_cast<int32_t*>(sKV + C::STAGES * C::KV_STAGE_BYTES);  // [topk]
  uint64_t* sMask = reinterpret_cast<uint64_t*>(sPhys + C::MAX_TILES * C::BN);   // [32]
  int32_t* sTiles = reinterpret_cast<int32_t*>(sMask + C::MAX_TILES);            // [32]
  float* sRed = reinterpret_cast<float*>(sTiles + C::MAX_TILES);        // [2][2][128]
  float* sLsum = sRed + 2 * 2 * 128;                            // [2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sLsum + 2 * 128);
  uint64_t* kv_full = bars;          // [2] 4 producer arrivals + gathered bytes
  uint64_t* kv_empty = bars + 2;     // [2] PV commit
  uint64_t* s_full = bars + 4;       // QK commit
  uint64_t* s_empty = bars + 5;      // 8 softmax warps
  uint64_t* p_full = bars + 6;       // 256 softmax threads
  uint64_t* pv_done = bars + 7;      // PV commit
  uint64_t* mx_bar = bars + 8;       // 256 arrivals per tile: both halves' partial max
  uint64_t* fin_bar = bars + 9;      // 256 arrivals: both halves' partial sums
  uint64_t* qk_fin = bars + 10;
  uint64_t* pv_fin = bars + 11;
  uint64_t* q_bar = bars + 12;       // 1 arrival + Q bytes
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int n_act_s;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int vh = static_cast<int>(blockIdx.x & 1u);   // value half
  const int split = blockIdx.y;
  const int r = blockIdx.x >> 1;
  const int row = p.row_begin + r;
  const int32_t* irow = p.idx + static_cast<int64_t>(r) * p.topk;
  const int n_tiles_all = p.topk / C::BN;

  // ---- row geometry
  int b, n_keys;
  int64_t key_base = 0;
  if (p.decode) {
    b = row;
    n_keys = min(p.seq_lens[b], p.max_seqlen);   // an entry above max_seqlen is a caller error
    key_base = static_cast<int64_t>(b) * p.kv_stride;
  } else {
    int lo = 0, hi = p.batch;
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (p.cu_seqlens[mid] <= row) lo = mid; else hi = mid;
    }
    b = lo;
    n_keys = row - p.cu_seqlens[lo] + 1;
    key_base = p.cu_seqlens[lo];
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(smem_u32(&kv_full[i]), 4);
      mbar_init(smem_u32(&kv_empty[i]), 1);
    }
    mbar_init(smem_u32(s_full), 1);
    mbar_init(smem_u32(s_empty), 8);
    mbar_init(smem_u32(p_full), 256);
    mbar_init(smem_u32(pv_done), 1);
    mbar_init(smem_u32(mx_bar), 256);
    mbar_init(smem_u32(fin_bar), 256);
    mbar_init(smem_u32(qk_fin), 1);
    mbar_init(smem_u32(pv_fin), 1);
    mbar_init(smem_u32(q_bar), 1);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(&tmem_base_s), C::TMEM_COLS);
  __syncthreads();
  if (threadIdx.x == 0) {
    // ---- Q: blocks [0, KBT) into the (still idle) gather ring, the rest into sQ
    tma_prefetch_desc(&kv_map);
    tma_prefetch_desc(&q_map);
    mbar_arrive_expect_tx(smem_u32(q_bar), C::KB_ALL * C::Q_KB_BYTES);
    for (int kb = 0; kb < C::KB_ALL; ++kb) {
      uint8_t* dst = kb < C::KBT ? sKV + kb * C::Q_KB_BYTES : sQ + (kb - C::KBT) * C::Q_KB_BYTES;
      tma_load_2d(smem_u32(dst), &q_map, smem_u32(q_bar), kb * 128, row * p.h);
    }
  }
  if (warp >= 12) {
    // ---- every selected key -> physical row (or -1), 16 keys per thread, loads in flight
    const int t = threadIdx.x - 384;
    for (int e = t; e < p.topk; e += 128) {
      const int v = irow[e];
      int64_t phys = -1;
      if (v >= 0 && v < n_keys) {
        if (p.decode && p.block_table != nullptr) {
          const int64_t id = __ldg(p.block_table + static_cast<int64_t>(b) * p.max_blocks +
                                   v / p.block_size);
          phys = id < 0 ? -1 : id * p.block_size + v % p.block_size;
        } else {
          phys = key_base + v;
        }
        if (phys >= p.num_kv_rows) phys = -1;
        if (phys < 0 && p.status) atomicOr(p.status, kStatusBadIndex);
      } else if (v >= n_keys && p.status) {
        atomicOr(p.status, kStatusBadIndex);
      }
      sPhys[e] = static_cast<int32_t>(phys);
    }
  }
  __syncthreads();
  if (warp >= 12) {
    // ---- per tile: the valid-key mask; invalid keys borrow the tile's first valid row
    for (int tt = warp - 12; tt < n_tiles_all; tt += 4) {
      int32_t* ph = sPhys + tt * C::BN;
      const int32_t a0 = ph[lane], a1 = ph[32 + lane];
      const uint32_t lo = __ballot_sync(0xffffffffu, a0 >= 0);
      const uint32_t hi = __ballot_sync(0xffffffffu, a1 >= 0);
      const uint64_t m = (static_cast<uint64_t>(hi) << 32) | lo;
      if (m != 0) {
        const int first = __ffsll(static_cast<long long>(m)) - 1;
        const int32_t fb = ph[first];
        __syncwarp();
        if (a0 < 0) ph[lane] = fb;
        if (a1 < 0) ph[32 + lane] = fb;
      }
      if (lane == 0) sMask[tt] = m;
    }
  }
  __syncthreads();
  if (warp == 0 && lane == 0) {
    // ---- the active tiles of this split, identical in both CTAs of the row
    int cnt = 0;
    for (int t = 0; t < n_tiles_all; ++t)
      if (sMask[t] != 0) {
        sTiles[cnt] = t;
        ++cnt;
      }
    const int per = (cnt + p.splits - 1) / p.splits;
    const int t0 = min(cnt, split * per);
    const int t1 = min(cnt, t0 + per);
    for (int i = t0; i < t1; ++i) sTiles[i - t0] = sTiles[i];
    n_act_s = t1 - t0;
  }
  if (warp >= 4 && warp < 12) {
    // ---- Q blocks [0, KBT) from the staging area into TMEM: head = lane, dim d in column
    // Q_COL + d / 2 (half h of the warps takes blocks h, h + 2, ...)
    const int hrow = (warp & 3) * 32 + lane;
    const int half = (warp - 4) >> 2;
    const uint32_t lane_addr = tmem_base_s + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(q_bar), 0, &abort_s))) {
      abort_s = 1;
      if (p.status) atomicOr(p.status, kStatusTimeout);
    } else {
      for (int kb = half; kb < C::KBT; kb += 2) {
        uint32_t u[32];
        const uint8_t* src = sKV + kb * C::Q_KB_BYTES;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + sw128_offset(hrow, ch));
          u[4 * ch + 0] = v.x;
          u[4 * ch + 1] = v.y;
          u[4 * ch + 2] = v.z;
          u[4 * ch + 3] = v.w;
        }
        tmem_st32(lane_addr + C::Q_COL + kb * 32, u);
      }
      tmem_wait_st();
    }
  }
  tc_fence_before();
  __syncthreads();   // the staging area is free for the gather ring from here on
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const int n = abort_s ? 0 : n_act_s;

  if (warp == 0) {
    // ------------------------------------------------------------ QK issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f32acc(1 /* bf16 */, 128, C::BN, 0, 0);
      const uint32_t qa = smem_u32(sQ);
      bool ok = n == 0 || mbar_wait(smem_u32(q_bar), 0, &abort_s);
      for (int i = 0; i < n && ok; ++i) {
        const int s = i % C::STAGES;
        ok = mbar_wait(smem_u32(&kv_full[s]), (i / C::STAGES) & 1, &abort_s);
        if (ok && i >= 1) ok = mbar_wait(smem_u32(s_empty), (i - 1) & 1, &abort_s);
        if (!ok) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(sKV + s * C::KV_STAGE_BYTES);
        for (int kb = 0; kb < C::KBT; ++kb)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16_ts(tmem + C::S_COL, tmem + C::Q_COL + kb * 32 + k * 8,
                         sdesc_sw128(ka + kb * C::KB_BYTES + k * 32, 16, 1024), idesc,
                         (kb | k) != 0);
        for (int kb = C::KBT; kb < C::KB_ALL; ++kb)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tmem + C::S_COL,
                      sdesc_sw128(qa + (kb - C::KBT) * C::Q_KB_BYTES + k * 32, 16, 1024),
                      sdesc_sw128(ka + kb * C::KB_BYTES + k * 32, 16, 1024), idesc, 1u);
        umma_commit(smem_u32(s_full));
      }
      if (!ok) {
        abort_s = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
      }
      umma_commit(smem_u32(qk_fin));
      mbar_wait(smem_u32(qk_fin), 0, nullptr);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ PV issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f32acc(1, 128, C::V_HALF, 0, 1);
      bool ok = true;
      for (int i = 0; i < n && ok; ++i) {
        const int s = i % C::STAGES;
        ok = mbar_wait(smem_u32(p_full), i & 1, &abort_s);
        if (!ok) break;
        tc_fence_after();
        const uint32_t va = smem_u32(sKV + s * C::KV_STAGE_BYTES) + vh * C::VKB * C::KB_BYTES;
#pragma unroll
        for (int k = 0; k < C::BN / 16; ++k)
          umma_bf16_ts(tmem, tmem + C::P_COL + k * 8,
                       sdesc_sw128(va + k * 16 * 128, C::KB_BYTES, 1024), idesc, (i | k) != 0);
        umma_commit(smem_u32(&kv_empty[s]));
        umma_commit(smem_u32(pv_done));
      }
      if (!ok) {
        abort_s = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
      }
      umma_commit(smem_u32(pv_fin));
      mbar_wait(smem_u32(pv_fin), 0, nullptr);
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ gather producers
    // Lane 0 of producer warp w gathers rows [16w, 16w + 16) of each tile: 4 rows x 64 dims
    // per TMA instruction, KB_ALL k-blocks.
    if (lane == 0) {
      const int pw = warp - 12;
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < n && ok; ++i) {
        const int s = i % C::STAGES;
        if (i >= C::STAGES)
          ok = mbar_wait(smem_u32(&kv_empty[s]), ((i / C::STAGES) - 1) & 1, &abort_s);
        if (!ok) break;
        const uint32_t bar = smem_u32(&kv_full[s]);
        mbar_arrive_expect_tx(bar, C::ROWS_PER_WARP_TX);
        const int32_t* ph = sPhys + sTiles[i] * C::BN + pw * 16;
        const uint32_t dst0 = smem_u32(sKV + s * C::KV_STAGE_BYTES) + pw * 16 * 128;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int4 rr = *reinterpret_cast<const int4*>(ph + 4 * g);
          for (int kb = 0; kb < C::KB_ALL; ++kb)
            tma_gather4(dst0 + kb * C::KB_BYTES + g * 512, &kv_map, bar, kb * 128, rr.x, rr.y,
                        rr.z, rr.w);
        }
        ++issued;
      }
      if (!ok) {
        abort_s = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
      }
      // no gather may still be writing this CTA's shared memory when it exits (immediate
      // unless the loop above was cut short)
      for (int i = max(0, issued - C::STAGES); i < issued; ++i)
        mbar_wait(smem_u32(&kv_full[i % C::STAGES]), (i / C::STAGES) & 1, nullptr);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int quad = warp & 3;
    const int half = (warp - 4) >> 2;           // keys [32 half, 32 half + 32) of each tile
    const int hrow = quad * 32 + lane;          // head = TMEM lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    constexpr int OC = C::V_HALF / 2;           // O columns this half rescales / stores
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = !abort_s;
    for (int i = 0; i < n && ok; ++i) {
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(s_full), i & 1, &abort_s));
      if (!ok) break;
      tc_fence_after();
      float sv[32];
      {
        uint32_t u[32];
        tmem_ld32(lane_addr + C::S_COL + half * 32, u);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[e] = __uint_as_float(u[e]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(s_empty));
      const uint32_t vbits = static_cast<uint32_t>(sMask[sTiles[i]] >> (32 * half));
      float m_half = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        sv[j] = ((vbits >> j) & 1u) ? sv[j] * p.scale_log2 : -INFINITY;
        m_half = fmaxf(m_half, sv[j]);
      }
      // row max over both halves (double-buffered by tile parity)
      float* red = sRed + (i & 1) * 256;
      red[half * 128 + hrow] = m_half;
      mbar_arrive(smem_u32(mx_bar));
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(mx_bar), i & 1, &abort_s));
      if (!ok) break;
      const float m_tile = fmaxf(red[hrow], red[128 + hrow]);
      // P and O are free once PV(i-1) has completed
      if (i >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(pv_done), (i - 1) & 1, &abort_s));
        if (!ok) break;
        tc_fence_after();
      }
      const bool need = m_tile > m_ref + 8.0f;
      float alpha = 1.f;
      if (need) {
        alpha = exp2f(m_ref - m_tile);
        l_sum *= alpha;
        m_ref = m_tile;
      }
      if (i >= 1 && __any_sync(0xffffffffu, need)) {
        for (int c0 = half * OC; c0 < (half + 1) * OC; c0 += 32) {
          uint32_t u[32];
          tmem_ld32(lane_addr + c0, u);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(__uint_as_float(u[j]) * alpha);
          tmem_st32(lane_addr + c0, u);
        }
      }
      uint32_t pk[16];
      float rowsum = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        // the denominator sums the fp32 probabilities; only the PV operand is rounded
        const float p0 = exp2f(sv[2 * e] - m_ref);
        const float p1 = exp2f(sv[2 * e + 1] - m_ref);
        rowsum += p0 + p1;
        const __nv_bfloat162 two = __floats2bfloat162_rn(p0, p1);
        pk[e] = *reinterpret_cast<const uint32_t*>(&two);
      }
      l_sum += rowsum;
      tmem_st16(lane_addr + C::P_COL + half * 16, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(p_full));
    }
    if (!ok) {
      abort_s = 1;
      if (p.status) atomicOr(p.status, kStatusTimeout);
    }
    // ---- epilogue: l = l(keys 0-31) + l(keys 32-63), the same order in both halves
    sLsum[half * 128 + hrow] = l_sum;
    mbar_arrive(smem_u32(fin_bar));
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(fin_bar), 0, &abort_s));
    const float l_tot = ok ? sLsum[hrow] + sLsum[128 + hrow] : 0.f;
    const bool write = hrow < p.h;
    const int64_t orow = static_cast<int64_t>(row) * p.h + hrow;
    if (ok && n > 0)
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(pv_done), (n - 1) & 1, &abort_s));
    tc_fence_after();
    const float inv_l = (n > 0 && l_tot > 0.f) ? 1.f / l_tot : 0.f;
    const float lse_v =
        (n > 0 && l_tot > 0.f) ? (m_ref + log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
    float* po = nullptr;
    if (p.part_o != nullptr)
      po = p.part_o + ((static_cast<int64_t>(split) * p.row_count + r) * p.h + hrow) * D_V +
           vh * C::V_HALF;
    for (int c0 = half * OC; c0 < (half + 1) * OC; c0 += 32) {
      float o[32];
      if (ok && n > 0) {
        uint32_t u[32];
        tmem_ld32(lane_addr + c0, u);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = __uint_as_float(u[j]) * inv_l;
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = 0.f;
      }
      if (!write) continue;
      if (po != nullptr) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(po + c0 + j) = make_float4(o[j], o[j + 1], o[j + 2], o[j + 3]);
      } else {
        __nv_bfloat16* dst = p.out + orow * D_V + vh * C::V_HALF + c0;
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 two = __floats2bfloat162_rn(o[j + 2 * e], o[j + 2 * e + 1]);
            pk[e] = *reinterpret_cast<const uint32_t*>(&two);
          }
          *reinterpret_cast<uint4*>(dst + j) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    if (write && vh == 0 && half == 0) {
      if (p.part_lse != nullptr)
        p.part_lse[(static_cast<int64_t>(split) * p.row_count + r) * p.h + hrow] = lse_v;
      else
        p.lse[orow] = lse_v;
    }
  }
  if (threadIdx.x == 0) mbar_wait(smem_u32(q_bar), 0, nullptr);   // Q has landed
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Merge split-KV partials by their LSE: O = sum_i e^(LSE_i - LSE) O_i, LSE = log sum e^LSE_i.
template <int D_V>
__global__ void __launch_bounds__(128) dsa_mla_combine_kernel(const MlaParams p) {
  const int r = blockIdx.x, hrow = blockIdx.y;
  const int64_t stride = static_cast<int64_t>(p.row_count) * p.h;
  const int64_t base = static_cast<int64_t>(r) * p.h + hrow;
  float m = -INFINITY;
  for (int s = 0; s < p.splits; ++s) m = fmaxf(m, p.part_lse[s * stride + base]);
  float wsum = 0.f;
  float wts[16];
  for (int s = 0; s < p.splits; ++s) {
    const float w = m == -INFINITY ? 0.f : expf(p.part_lse[s * stride + base] - m);
    wts[s] = w;
    wsum += w;
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  const int64_t orow = static_cast<int64_t>(p.row_begin + r) * p.h + hrow;
  for (int d = threadIdx.x * 4; d < D_V; d += 128 * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < p.splits; ++s) {
      const float4 v = *reinterpret_cast<const float4*>(p.part_o + (s * stride + base) * D_V + d);
      const float w = wts[s] * inv;
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
    const __nv_bfloat162 a = __floats2bfloat162_rn(acc.x, acc.y);
    const __nv_bfloat162 c = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&a);
    pk.y = *reinterpret_cast<const uint32_t*>(&c);
    *reinterpret_cast<uint2*>(p.out + orow * D_V + d) = pk;
  }
  if (threadIdx.x == 0) p.lse[orow] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

}  // namespace dsa
