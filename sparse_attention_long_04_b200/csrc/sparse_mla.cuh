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
//   (invalid keys borrow a valid row of their tile and are masked out of the softmax).  The
//   rows of each 64-key tile are gathered with 16-byte cp.async in two parts with their own
//   2-slot rings: the value dims of this CTA (needed until PV) and the other dims (needed only
//   by QK, so refilled as soon as QK is done); each copying thread's arrival on the slot's
//   barrier fires when its copies land, so no producer waits on memory.  Per tile:
//   S = Q K^T (tcgen05 bf16, M = 128 heads, N = 64 keys, fp32 in TMEM), an online softmax
//   (thread = head = TMEM lane, all 64 keys), P (bf16) back into TMEM, and O_v += P V_v
//   (A = P from TMEM, N = D_V/2, V read MN-major straight out of the gathered tile).  Rescaling
//   of O is lazy (only when a tile's max beats the running reference by more than 2^8, so
//   P <= 256).
// TMEM columns: O [0, D_V/2) | S [+64) | P [+32) | Q (KBT x 32 columns).
// Warp roles per CTA (512 threads): warp 0 loads Q and issues QK, warp 2 issues PV, warp 1
// owns TMEM, warps 4-7 move Q into TMEM, run the softmax and the epilogue, warps 8-15 resolve
// the keys, then gather rows [16w, 16w + 16) of every tile: warps 8-11 the QK-only dims,
// warps 12-15 the value dims.  Grid: x = 2 * row + v, y = split-KV slice.
// Without an index array the selection is every prior key (dense causal attention), which is
// what the top-k keeps whenever a row has at most topk prior keys.  A dense row with more keys
// than topk (prefill only: its keys are consecutive packed rows) is streamed: its tiles, their
// valid-key masks and physical rows are computed on the fly instead of resolved up front.
//
// Target mode (kTarget): the indexer's training target on the same selection, the main
// attention's distribution summed over heads and normalised ("DeepSeek V3.2-Exp Cuts
// Long-Context Costs with DeepSeek Sparse Attention (DSA)", "Training signal"):
//   target[t, e] = (1/H) sum_h exp(sigma q[t,h,:] . kv[idx[t,e], :] - LSE[t,h])
// with the LSE of the forward pass over the same selection.  The gathers and the QK product
// are the forward's; there is no PV.  The two CTAs of a row take alternate tiles (each gathers
// every dim of its tiles), the QK commit frees both parts of a slot, and the softmax warps
// turn each logit into its probability (thread = head), sum the 128 heads of every key with a
// butterfly across lanes and a 4-warp pass through shared memory, and write the 64 targets of
// the tile.  Entries with idx = -1 get 0.
#pragma once
#include <type_traits>

#include "sm100.cuh"

namespace dsa {

struct MlaParams {
  const __nv_bfloat16* q;      // [T, H, D_QK]
  const __nv_bfloat16* kv;     // [R, D_QK]
  const int32_t* idx;          // [row_count, topk], relative to row_begin; null: dense
                               // (every prior key; the caller guarantees pos + 1 <= topk)
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
  const float* lse_in;         // target mode: the forward's LSE [T, H]
  float* target;               // target mode: [row_count, ld_target], relative to row_begin
  int64_t ld_target;           // target mode: row stride (topk; dense: >= the longest row)
};

template <int D_QK, int D_V>
struct MlaCfg {
  static constexpr int KB_ALL = (D_QK + 63) / 64;     // 64-element k-blocks of a latent row
  static constexpr int V_HALF = D_V / 2;              // value dims per CTA
  static constexpr int VKB = V_HALF / 64;             // value k-blocks per CTA
  static constexpr int KK = KB_ALL - VKB;             // QK-only k-blocks
  static constexpr int BN = 64;                       // keys per tile
  static constexpr int STAGES = 2;
  static constexpr int PREFETCH = 3;                  // tiles ahead whose rows go to L2
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
  static constexpr int K_SLOT_BYTES = KK * KB_BYTES;
  static constexpr int V_SLOT_BYTES = VKB * KB_BYTES;
  static constexpr int RING_BYTES = STAGES * (K_SLOT_BYTES + V_SLOT_BYTES);
  static constexpr int Q_KB_BYTES = 128 * 128;                        // one k-block of Q
  static constexpr int Q_SMEM_BYTES = KBS * Q_KB_BYTES;
  static constexpr int RED_BYTES = 2 * 4 * BN * 4;                    // target mode
  static constexpr int SMEM_USED = 1024 + Q_SMEM_BYTES + RING_BYTES + MAX_TILES * BN * 4 +
                                   MAX_TILES * 12 + 256 + RED_BYTES;
  // at least 116 KB, so that one CTA runs per SM (its TMEM allocation never waits)
  static constexpr int SMEM_BYTES = SMEM_USED > 116 * 1024 ? SMEM_USED : 116 * 1024;
  static_assert(V_HALF % 64 == 0 && V_HALF <= 256, "PV MMA N");
  static_assert(Q_COL + KBT * 32 <= 512, "TMEM columns");
  static_assert(KBT * Q_KB_BYTES <= RING_BYTES, "Q staging fits the gather rings");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <int D_QK, int D_V, bool kTarget = false>
__global__ void __launch_bounds__(512, 1)
    dsa_sparse_mla_kernel(const __grid_constant__ CUtensorMap q_map, const MlaParams p) {
  using C = MlaCfg<D_QK, D_V>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                                           // [KBS][128 heads][128 B]
  uint8_t* sRing = sQ + C::Q_SMEM_BYTES;                        // gather rings (Q staging first)
  uint8_t* sK = sRing;                                          // [STAGES][KK k-blocks]
  uint8_t* sV = sRing + C::STAGES * C::K_SLOT_BYTES;            // [STAGES][VKB k-blocks]
  int32_t* sPhys = reinterpret_cast<int32_t*>(sRing + C::RING_BYTES);             // [topk]
  uint64_t* sMask = reinterpret_cast<uint64_t*>(sPhys + C::MAX_TILES * C::BN);   // [32]
  int32_t* sTiles = reinterpret_cast<int32_t*>(sMask + C::MAX_TILES);            // [32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sTiles + C::MAX_TILES);
  uint64_t* k_full = bars;           // [2] 128 K-part threads (each when its copies land)
  uint64_t* k_empty = bars + 2;      // [2] QK commit
  uint64_t* v_full = bars + 4;       // [2] 128 V-part threads (each when its copies land)
  uint64_t* v_empty = bars + 6;      // [2] PV commit
  uint64_t* s_full = bars + 8;       // QK commit
  uint64_t* s_empty = bars + 9;      // 4 softmax warps
  uint64_t* p_full = bars + 10;      // 128 softmax threads
  uint64_t* pv_done = bars + 11;     // PV commit
  uint64_t* qk_fin = bars + 12;
  uint64_t* pv_fin = bars + 13;
  uint64_t* q_bar = bars + 14;       // 1 arrival + Q bytes
  uint64_t* red_full = bars + 15;    // [2] target mode: 4 softmax warps
  uint64_t* red_empty = bars + 17;   // [2] target mode: the writing warp
  float* sRed = reinterpret_cast<float*>(bars + 32);   // target mode: [2][4 warps][BN]
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int n_act_s;

  wait_prior_grid();   // (launched early: the indices come from the previous kernel)
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int vh = static_cast<int>(blockIdx.x & 1u);   // value half
  const int split = blockIdx.y;
  const int r = blockIdx.x >> 1;
  const int row = p.row_begin + r;
  const bool dense = p.idx == nullptr;
  const int32_t* irow = dense ? nullptr : p.idx + static_cast<int64_t>(r) * p.topk;
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

  // a dense prefill row longer than the resolved-key arrays: tiles computed on the fly
  const bool stream_dense = dense && !p.decode && n_keys > p.topk;
  __shared__ int t0_s;
  auto tile_at = [&](int i) -> int {
    return stream_dense ? t0_s + (kTarget ? 2 * i + vh : i) : sTiles[i];
  };
  auto mask_of = [&](int t) -> uint64_t {
    if (!stream_dense) return sMask[t];
    const int rem = n_keys - t * C::BN;
    return rem >= C::BN ? ~0ull : ((1ull << rem) - 1ull);
  };

  // the selected keys' indices (8 per thread of warps 8-15), loaded before the set-up and the Q
  // load, so that their latency overlaps both
  constexpr int KPT = C::MAX_TILES * C::BN / 256;
  int v[KPT];
  if (warp >= 8 && !stream_dense) {
    const int t = threadIdx.x - 256;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      const int e = t + 256 * j;
      v[j] = e >= p.topk ? -1 : dense ? (e < n_keys ? e : -1) : irow[e];
    }
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(smem_u32(&k_full[i]), 128);
      mbar_init(smem_u32(&k_empty[i]), 1);
      mbar_init(smem_u32(&v_full[i]), 128);
      mbar_init(smem_u32(&v_empty[i]), 1);
    }
    mbar_init(smem_u32(s_full), 1);
    mbar_init(smem_u32(s_empty), 4);
    mbar_init(smem_u32(p_full), 128);
    mbar_init(smem_u32(pv_done), 1);
    mbar_init(smem_u32(qk_fin), 1);
    mbar_init(smem_u32(pv_fin), 1);
    mbar_init(smem_u32(q_bar), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&red_full[i]), 4);
      mbar_init(smem_u32(&red_empty[i]), 1);
    }
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(&tmem_base_s), C::TMEM_COLS);
  __syncthreads();
  if (threadIdx.x == 0) {
    // ---- Q: blocks [0, KBT) into the (still idle) gather rings, the rest into sQ
    tma_prefetch_desc(&q_map);
    mbar_arrive_expect_tx(smem_u32(q_bar), C::KB_ALL * C::Q_KB_BYTES);
    for (int kb = 0; kb < C::KB_ALL; ++kb) {
      uint8_t* dst = kb < C::KBT ? sRing + kb * C::Q_KB_BYTES : sQ + (kb - C::KBT) * C::Q_KB_BYTES;
      tma_load_2d(smem_u32(dst), &q_map, smem_u32(q_bar), kb * 128, row * p.h);
    }
  }
  if (warp >= 8 && !stream_dense) {
    // ---- every selected key -> physical row (or -1): the indices loaded above, then all
    // block-table loads in flight together
    const int t = threadIdx.x - 256;
    int64_t phys[KPT];
    bool bad_idx = false;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      phys[j] = -1;
      if (v[j] >= n_keys) bad_idx = true;
      if (v[j] >= 0 && v[j] < n_keys) {
        if (p.decode && p.block_table != nullptr)
          phys[j] = __ldg(p.block_table + static_cast<int64_t>(b) * p.max_blocks +
                          v[j] / p.block_size);
        else
          phys[j] = key_base + v[j];
      }
    }
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      int64_t ph = phys[j];
      if (v[j] >= 0 && v[j] < n_keys) {
        if (p.decode && p.block_table != nullptr)
          ph = ph < 0 ? -1 : ph * p.block_size + v[j] % p.block_size;
        if (ph >= p.num_kv_rows) ph = -1;
        if (ph < 0) bad_idx = true;
      }
      const int e = t + 256 * j;
      if (e < p.topk) sPhys[e] = static_cast<int32_t>(ph);
    }
    if (bad_idx && p.status) atomicOr(p.status, kStatusBadIndex);
  }
  __syncthreads();
  if (warp >= 8 && !stream_dense) {
    // ---- per tile: the valid-key mask; invalid keys borrow the tile's first valid row
    for (int tt = warp - 8; tt < n_tiles_all; tt += 8) {
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
      if (kTarget && m == 0 && vh == 0 && split == 0 &&   // no valid key: targets are 0
          static_cast<int64_t>(tt + 1) * C::BN <= p.ld_target) {
        float* tg = p.target + static_cast<int64_t>(r) * p.ld_target + tt * C::BN;
        tg[lane] = 0.f;
        tg[32 + lane] = 0.f;
      }
    }
  }
  __syncthreads();
  if (warp == 0 && lane == 0) {
    // ---- the active tiles of this split, identical in both CTAs of the row
    int cnt = 0;
    if (stream_dense) {
      cnt = (n_keys + C::BN - 1) / C::BN;
    } else {
      for (int t = 0; t < n_tiles_all; ++t)
        if (sMask[t] != 0) {
          sTiles[cnt] = t;
          ++cnt;
        }
    }
    const int per = (cnt + p.splits - 1) / p.splits;
    const int t0 = min(cnt, split * per);
    const int t1 = min(cnt, t0 + per);
    int m = 0;   // target mode: the two CTAs of a row take alternate tiles
    if (stream_dense) {
      t0_s = t0;
      m = kTarget ? (t1 - t0 - vh + 1) / 2 : t1 - t0;
      if (m < 0) m = 0;
    } else {
      for (int i = t0; i < t1; ++i)
        if (!kTarget || ((i - t0) & 1) == vh) sTiles[m++] = sTiles[i];
    }
    n_act_s = m;
  }
  if (warp >= 4 && warp < 8) {
    // ---- Q blocks [0, KBT) from the staging area into TMEM: head = lane, dim d in column
    // Q_COL + d / 2
    const int hrow = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = tmem_base_s + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    if (!(warp_mbar_wait(smem_u32(q_bar), 0, &abort_s))) {
      abort_s = 1;
      if (p.status) atomicOr(p.status, kStatusTimeout);
    } else {
      for (int kb = 0; kb < C::KBT; ++kb) {
        uint32_t u[32];
        const uint8_t* src = sRing + kb * C::Q_KB_BYTES;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 q4 = *reinterpret_cast<const uint4*>(src + sw128_offset(hrow, ch));
          u[4 * ch + 0] = q4.x;
          u[4 * ch + 1] = q4.y;
          u[4 * ch + 2] = q4.z;
          u[4 * ch + 3] = q4.w;
        }
        tmem_st32(lane_addr + C::Q_COL + kb * 32, u);
      }
      tmem_wait_st();
    }
  }
  tc_fence_before();
  __syncthreads();   // the staging area is free for the gather rings from here on
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const int n = abort_s ? 0 : n_act_s;

  if (warp == 0) {
    // ------------------------------------------------------------ QK issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f32acc(1 /* bf16 */, 128, C::BN, 0, 0);
      const uint32_t qa = smem_u32(sQ);
      const int v0 = vh * C::VKB;                 // first value k-block of this CTA
      bool ok = n == 0 || mbar_wait(smem_u32(q_bar), 0, &abort_s);
      for (int i = 0; i < n && ok; ++i) {
        const int s = i % C::STAGES;
        const uint32_t ph = (i / C::STAGES) & 1;
        ok = mbar_wait(smem_u32(&k_full[s]), ph, &abort_s) &&
             mbar_wait(smem_u32(&v_full[s]), ph, &abort_s);
        if (ok && i >= 1) ok = mbar_wait(smem_u32(s_empty), (i - 1) & 1, &abort_s);
        if (!ok) break;
        tc_fence_after();
        fence_proxy_async_smem();   // the gathered rows were written by cp.async
        const uint32_t ka = smem_u32(sK + s * C::K_SLOT_BYTES);
        const uint32_t va = smem_u32(sV + s * C::V_SLOT_BYTES);
        // k-block kb of the tile: a value block of this CTA in the V slot, else the K slot
        auto kb_addr = [&](int kb) -> uint32_t {
          if (kb >= v0 && kb < v0 + C::VKB) return va + (kb - v0) * C::KB_BYTES;
          return ka + (kb < v0 ? kb : kb - C::VKB) * C::KB_BYTES;
        };
        for (int kb = 0; kb < C::KBT; ++kb) {
          const uint32_t ba = kb_addr(kb);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16_ts(tmem + C::S_COL, tmem + C::Q_COL + kb * 32 + k * 8,
                         sdesc_sw128(ba + k * 32, 16, 1024), idesc, (kb | k) != 0);
        }
        for (int kb = C::KBT; kb < C::KB_ALL; ++kb) {
          const uint32_t ba = kb_addr(kb);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tmem + C::S_COL,
                      sdesc_sw128(qa + (kb - C::KBT) * C::Q_KB_BYTES + k * 32, 16, 1024),
                      sdesc_sw128(ba + k * 32, 16, 1024), idesc, 1u);
        }
        umma_commit(smem_u32(s_full));
        umma_commit(smem_u32(&k_empty[s]));
        if (kTarget) umma_commit(smem_u32(&v_empty[s]));   // no PV reads the slot
      }
      if (!ok) {
        abort_s = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
      }
      umma_commit(smem_u32(qk_fin));
      mbar_wait(smem_u32(qk_fin), 0, nullptr);
    }
  } else if (warp == 2 && !kTarget) {
    // ------------------------------------------------------------ PV issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f32acc(1, 128, C::V_HALF, 0, 1);
      bool ok = true;
      for (int i = 0; i < n && ok; ++i) {
        const int s = i % C::STAGES;
        ok = mbar_wait(smem_u32(p_full), i & 1, &abort_s);
        if (!ok) break;
        tc_fence_after();
        const uint32_t va = smem_u32(sV + s * C::V_SLOT_BYTES);
#pragma unroll
        for (int k = 0; k < C::BN / 16; ++k)
          umma_bf16_ts(tmem, tmem + C::P_COL + k * 8,
                       sdesc_sw128(va + k * 16 * 128, C::KB_BYTES, 1024), idesc, (i | k) != 0);
        umma_commit(smem_u32(&v_empty[s]));
        umma_commit(smem_u32(pv_done));
      }
      if (!ok) {
        abort_s = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
      }
      umma_commit(smem_u32(pv_fin));
      mbar_wait(smem_u32(pv_fin), 0, nullptr);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ gather producers
    // Warp 8 + 4 part + w copies rows [16w, 16w + 16) of each tile: part 0 the QK-only k-blocks
    // (K slot), part 1 this CTA's value k-blocks (V slot), 16-byte cp.async per lane; each lane
    // then arrives on the slot's full barrier once its copies have landed.
    const int part = (warp - 8) >> 2;
    const int pw = (warp - 8) & 3;
    const int ch = lane & 7;                    // 16-byte chunk of a 128-byte row block
    const int rsub = lane >> 3;                 // rows rsub, rsub + 4, rsub + 8, rsub + 12
    uint64_t* full = part == 0 ? k_full : v_full;
    uint64_t* empty = part == 0 ? k_empty : v_empty;
    // one tile's part: rows [16 pw, 16 pw + 16), NKB k-blocks (latent-row block kb_of(ks))
    auto copy_part = [&](auto nkb_c, uint8_t* dst, auto phys_of, auto kb_of) {
      constexpr int NKB = decltype(nkb_c)::value;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int rr = rsub + 4 * j;
        const __nv_bfloat16* src = p.kv + phys_of(rr) * D_QK + ch * 8;
        const uint32_t drow = smem_u32(dst) + sw128_offset(pw * 16 + rr, ch);
#pragma unroll
        for (int ks = 0; ks < NKB; ++ks) {
          const int kb = kb_of(ks);
          const bool in = kb * 64 + ch * 8 < D_QK;
          cp_async_16(drow + ks * C::KB_BYTES, in ? static_cast<const void*>(src + kb * 64)
                                                  : static_cast<const void*>(p.kv),
                      in ? 16u : 0u);
        }
      }
    };
    bool ok = true;
    for (int i = 0; i < n && ok; ++i) {
      const int s = i % C::STAGES;
      if (i >= C::STAGES &&
          !(warp_mbar_wait(smem_u32(&empty[s]), ((i / C::STAGES) - 1) & 1,
                                             &abort_s))) {
        ok = false;
        break;
      }
      const int tile = tile_at(i);
      const int32_t* ph = sPhys + tile * C::BN + pw * 16;
      // physical row of row rr of this warp's 16: resolved up front, or (streamed dense rows)
      // consecutive packed rows, keys past the row borrowing the tile's first key
      auto phys_of = [&](int rr) -> int64_t {
        if (!stream_dense) return ph[rr];
        const int key = tile * C::BN + pw * 16 + rr;
        return key_base + (key < n_keys ? key : tile * C::BN);
      };
      if (part == 0)   // the QK-only k-blocks: all but this CTA's value blocks
        copy_part(std::integral_constant<int, C::KK>{}, sK + s * C::K_SLOT_BYTES, phys_of,
                  [&](int ks) { return ks < vh * C::VKB ? ks : ks + C::VKB; });
      else             // this CTA's value k-blocks
        copy_part(std::integral_constant<int, C::VKB>{}, sV + s * C::V_SLOT_BYTES, phys_of,
                  [&](int ks) { return vh * C::VKB + ks; });
      cp_async_arrive_noinc(smem_u32(&full[s]));
      // the rows of the tile PREFETCH steps ahead into L2 (its slot is not free yet): one
      // thread per row of the K-part warps, each CTA of the pair half of the row, so that the
      // gather of that tile reads L2 instead of HBM
      if (part == 0 && i + C::PREFETCH < n) {
        const int t2 = tile_at(i + C::PREFETCH);
        const int rr = (warp - 8) * 32 + lane;      // 0..127: rows 0..63 only
        if (rr < C::BN) {
          int64_t row2;
          if (!stream_dense) {
            row2 = sPhys[t2 * C::BN + rr];
          } else {
            const int key = t2 * C::BN + rr;
            row2 = key_base + (key < n_keys ? key : t2 * C::BN);
          }
          constexpr uint32_t kHalf = (D_QK * 2 / 2 + 15) / 16 * 16;
          const uint32_t off = vh * kHalf;
          const uint32_t bytes = vh == 0 ? kHalf : D_QK * 2 - kHalf;
          if (bytes > 0)
            prefetch_l2(reinterpret_cast<const uint8_t*>(p.kv + row2 * D_QK) + off, bytes);
        }
      }
    }
    if (!ok) {
      abort_s = 1;
      if (p.status) atomicOr(p.status, kStatusTimeout);
    }
    cp_async_wait_all();   // nothing may still be writing this CTA's shared memory at exit
  } else if (kTarget && warp >= 4) {
    // ------------------------------------------------------------ target: p per head, head sum
    const int w4 = warp & 3;
    const int hrow = w4 * 32 + lane;            // head = TMEM lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(w4 * 32) << 16);
    // heads past H (the small shapes run 128 MMA rows for fewer heads) contribute nothing
    const float lse2 =
        hrow < p.h ? p.lse_in[static_cast<int64_t>(row) * p.h + hrow] * 1.4426950408889634f
                   : INFINITY;
    // after the butterfly this lane holds the head sums of keys key0 and key0 + 1
    const int key0 = warp_sum64_first(lane);
    const float inv_h = 1.f / static_cast<float>(p.h);
    const float sc = p.scale_log2;
    bool ok = !abort_s;
    for (int i = 0; i < n && ok; ++i) {
      ok = (warp_mbar_wait(smem_u32(s_full), i & 1, &abort_s));
      if (!ok) break;
      tc_fence_after();
      uint32_t su[2][32];
      tmem_ld32(lane_addr + C::S_COL, su[0]);
      tmem_ld32(lane_addr + C::S_COL + 32, su[1]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(s_empty));
      const uint64_t vmask = mask_of(tile_at(i));
      float v[64];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint32_t vb = static_cast<uint32_t>(vmask >> (32 * hh));
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float pr = exp2f(fmaf(__uint_as_float(su[hh][j]), sc, -lse2));
          v[32 * hh + j] = ((vb >> j) & 1u) ? pr : 0.f;
        }
      }
      warp_sum64(v, lane);
      // the 4 warps' sums meet in shared memory (double-buffered by tile parity)
      const int buf = i & 1;
      float* red = sRed + buf * 4 * C::BN;
      if (i >= 2) {
        ok = (warp_mbar_wait(smem_u32(&red_empty[buf]), ((i >> 1) - 1) & 1, &abort_s));
        if (!ok) break;
      }
      *reinterpret_cast<float2*>(red + w4 * C::BN + key0) = make_float2(v[0], v[1]);
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&red_full[buf]));
      if (w4 == 0) {
        ok = (warp_mbar_wait(smem_u32(&red_full[buf]), (i >> 1) & 1, &abort_s));
        if (!ok) break;
        float* tg = p.target + static_cast<int64_t>(r) * p.ld_target + tile_at(i) * C::BN;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int e = lane + 32 * c;
          tg[e] = ((red[e] + red[C::BN + e]) + (red[2 * C::BN + e] + red[3 * C::BN + e])) * inv_h;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&red_empty[buf]));
      }
    }
    if (!ok) {
      abort_s = 1;
      if (p.status) atomicOr(p.status, kStatusTimeout);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int hrow = (warp & 3) * 32 + lane;    // head = TMEM lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = !abort_s;
    for (int i = 0; i < n && ok; ++i) {
      ok = (warp_mbar_wait(smem_u32(s_full), i & 1, &abort_s));
      if (!ok) break;
      tc_fence_after();
      uint32_t su[2][32];                       // S of keys [32 hh, 32 hh + 32)
      tmem_ld32(lane_addr + C::S_COL, su[0]);
      tmem_ld32(lane_addr + C::S_COL + 32, su[1]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(s_empty));
      const uint64_t vmask = mask_of(tile_at(i));
      // the tile max of the unscaled logits (sigma log2 e > 0), as 8 independent partial maxima
      float mm[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mm[q] = -INFINITY;
      if (vmask == ~0ull) {                     // every key of the tile is valid (the usual case)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int j = 0; j < 32; ++j) mm[j & 7] = fmaxf(mm[j & 7], __uint_as_float(su[hh][j]));
      } else {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t vb = static_cast<uint32_t>(vmask >> (32 * hh));
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float x = ((vb >> j) & 1u) ? __uint_as_float(su[hh][j]) : -INFINITY;
            su[hh][j] = __float_as_uint(x);    // invalid keys: -inf, so p = 0 below
            mm[j & 7] = fmaxf(mm[j & 7], x);
          }
        }
      }
      const float m_tile =
          fmaxf(fmaxf(fmaxf(mm[0], mm[1]), fmaxf(mm[2], mm[3])),
                fmaxf(fmaxf(mm[4], mm[5]), fmaxf(mm[6], mm[7]))) * p.scale_log2;
      // P and O are free once PV(i-1) has completed
      if (i >= 1) {
        ok = (warp_mbar_wait(smem_u32(pv_done), (i - 1) & 1, &abort_s));
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
      // p = 2^(sigma log2e s - m_ref) (0 for invalid keys); 8 independent partial sums
      float rs[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) rs[q] = 0.f;
      const float sc = p.scale_log2, nm = -m_ref;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          // the denominator sums the fp32 probabilities; only the PV operand is rounded
          const float p0 = exp2f(fmaf(__uint_as_float(su[hh][2 * e]), sc, nm));
          const float p1 = exp2f(fmaf(__uint_as_float(su[hh][2 * e + 1]), sc, nm));
          rs[(2 * e) & 7] += p0;
          rs[(2 * e + 1) & 7] += p1;
          const __nv_bfloat162 two = __floats2bfloat162_rn(p0, p1);
          pk[e] = *reinterpret_cast<const uint32_t*>(&two);
        }
        tmem_st16(lane_addr + C::P_COL + hh * 16, pk);
      }
      const float rowsum = ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
      l_sum += rowsum;
      // O to the new reference (after P, so the logits are no longer live; before PV(i))
      if (i >= 1 && __any_sync(0xffffffffu, need)) {
        for (int c0 = 0; c0 < C::V_HALF; c0 += 32) {
          uint32_t u[32];
          tmem_ld32(lane_addr + c0, u);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(__uint_as_float(u[j]) * alpha);
          tmem_st32(lane_addr + c0, u);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(p_full));
    }
    if (!ok) {
      abort_s = 1;
      if (p.status) atomicOr(p.status, kStatusTimeout);
    }
    // ---- epilogue
    const bool write = hrow < p.h;
    const int64_t orow = static_cast<int64_t>(row) * p.h + hrow;
    if (ok && n > 0)
      ok = (warp_mbar_wait(smem_u32(pv_done), (n - 1) & 1, &abort_s));
    tc_fence_after();
    const float inv_l = (ok && n > 0 && l_sum > 0.f) ? 1.f / l_sum : 0.f;
    const float lse_v =
        (ok && n > 0 && l_sum > 0.f) ? (m_ref + log2f(l_sum)) * 0.69314718055994531f : -INFINITY;
    float* po = nullptr;
    if (p.part_o != nullptr)
      po = p.part_o + ((static_cast<int64_t>(split) * p.row_count + r) * p.h + hrow) * D_V +
           vh * C::V_HALF;
    for (int c0 = 0; c0 < C::V_HALF; c0 += 32) {
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
    if (write && vh == 0) {
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
