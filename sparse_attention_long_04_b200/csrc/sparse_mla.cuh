// Sparse MLA attention in MQA mode (stage 3) and the split-KV combine.
//
// For query row t, head h, over the selected logical keys I_t (idx >= 0):
//   l_s = sigma * q[t,h,:] . kv[s,:]            (all D_QK = latent + RoPE dims)
//   O[t,h,:] = sum_s softmax(l)_s * kv[s, 0:D_V] (values = the first D_V latent dims)
//   LSE[t,h] = log sum_s exp(l_s)
// Every selected latent row is shared by all query heads ("MLA in MQA mode ... each latent KV
// entry is shared across query heads", "DeepSeek V3.2-Exp Cuts Long-Context Costs with
// DeepSeek Sparse Attention (DSA)", "Instantiation").
//
// Design (sm_100a).  O for 128 heads x 512 values in fp32 is 256 KB = all of one SM's TMEM,
// and Q (128 x 576 bf16 = 144 KB) plus gathered tiles do not fit one CTA's shared memory, so
// each query row runs on a 2-CTA cluster:
//   CTA r owns the QK dims D_r (r = 0: [0, D_V/2); r = 1: [D_V/2, D_QK)) and the value dims
//   [r D_V/2, (r+1) D_V/2).  Its slice of Q lives in Tensor Memory as the A operand of the QK
//   MMA; the selected latent rows are gathered (their D_r dims) into 128-byte-swizzled shared
//   memory tiles of 64 keys.  Per tile: S_r = Q_r K_r^T (tcgen05 bf16, A from TMEM, M = 128
//   heads, N = 64 keys); the two CTAs swap S_r with bulk shared-to-shared copies into each
//   other's memory and both form S = S_0 + S_1 in the same order, so both run an identical
//   online softmax; P goes to TMEM and CTA r accumulates O_r += P V_r (A = P from TMEM,
//   N = D_V/2, K = 64 keys, V read MN-major straight out of the gathered tile).  No tensor
//   work is duplicated.  Rescaling of O is lazy (only when a tile's max beats the running
//   reference by more than 2^8, so P <= 256).
// TMEM columns: O [0, V_HALF) | S [V_HALF, +64) | P [+64, +32) | Q (kb_count x 32 columns).
// Warp roles per CTA (512 threads): warp 0 issues QK, warp 2 issues PV, warp 1 owns TMEM and
// forwards read signals to the peer, warp 3 copies our partial logits to the peer,
// warps 4-11 run the softmax (thread = head = TMEM lane; warps 4-7 take keys 0-31 of a tile,
// warps 8-11 keys 32-63) and the epilogue, warps 12-15 resolve indices and gather rows with
// 16-byte cp.async (3 stages).  Grid: x = 2 * row (the cluster pair), y = split-KV slice.
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
  static constexpr int V_HALF = D_V / 2;
  static constexpr int VKB = V_HALF / 64;             // value k-blocks per CTA
  static constexpr int KBC = KB_ALL - VKB;            // k-blocks held by rank 1 (>= rank 0)
  static constexpr int BN = 64;                       // keys per tile
  static constexpr int STAGES = 3;
  static constexpr int MAX_TILES = 32;                // topk <= 2048
  static constexpr int THREADS = 512;
  static constexpr int KV_STAGE_BYTES = KBC * BN * 128;
  static constexpr int X_BYTES = 128 * BN * 4;        // partial logits of one tile
  static constexpr int S_COL = V_HALF;
  static constexpr int P_COL = S_COL + BN;
  static constexpr int Q_COL = P_COL + BN / 2;
  static constexpr int TMEM_NEED = Q_COL + KBC * 32;
  static constexpr int TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
  static constexpr int SMEM_BYTES = 1024 + STAGES * KV_STAGE_BYTES + 3 * X_BYTES +
                                    STAGES * 8 + MAX_TILES * 12 +
                                    2 * 2 * 128 * 4 + 2 * 128 * 4 + 512;
  static_assert(KBC >= VKB, "rank 1 holds at least as many k-blocks as rank 0");
  static_assert(V_HALF % 64 == 0 && V_HALF <= 256, "PV MMA N");
  static_assert(TMEM_NEED <= 512, "TMEM columns");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(SMEM_BYTES > 114 * 1024, "one CTA per SM (TMEM and cluster peers)");
};

template <int D_QK, int D_V>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(512, 1)
    dsa_sparse_mla_kernel(const MlaParams p) {
  using C = MlaCfg<D_QK, D_V>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sKV = smem;                                          // [STAGES] gathered tiles
  uint8_t* sXin = sKV + C::STAGES * C::KV_STAGE_BYTES;          // [2] peer's partial logits
  uint8_t* sXout = sXin + 2 * C::X_BYTES;                       // ours, staged for the copy
  // [STAGES][4]: per producer warp, its 16 rows whose cache location was invalid
  uint16_t* sBad = reinterpret_cast<uint16_t*>(sXout + C::X_BYTES);
  uint64_t* sMask = reinterpret_cast<uint64_t*>(sBad + C::STAGES * 4);   // [32] valid keys

  int32_t* sTiles = reinterpret_cast<int32_t*>(sMask + C::MAX_TILES);   // [32] active tiles
  float* sRed = reinterpret_cast<float*>(sTiles + C::MAX_TILES);        // [2][2][128]
  float* sLsum = sRed + 2 * 2 * 128;                            // [2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sLsum + 2 * 128);
  uint64_t* kv_full = bars;          // [3] 128 producer arrivals
  uint64_t* kv_empty = bars + 3;     // [3] QK commit + PV commit
  uint64_t* s_full = bars + 6;       // QK commit
  uint64_t* s_empty = bars + 7;      // 8 softmax warps
  uint64_t* p_full = bars + 8;       // 256 softmax threads
  uint64_t* pv_done = bars + 9;      // PV commit
  uint64_t* x_full = bars + 10;      // [2] 1 local arrive + X_BYTES from the peer's copy
  uint64_t* peer_free = bars + 12;   // [2] 1 remote arrival: the peer read that buffer
  uint64_t* mx_bar = bars + 14;      // 256 arrivals per tile: both halves' partial max
  uint64_t* fin_bar = bars + 15;     // 256 arrivals: both halves' partial sums
  uint64_t* qk_fin = bars + 16;
  uint64_t* pv_fin = bars + 17;
  uint64_t* staged = bars + 18;      // 256 arrivals: our partial logits are staged
  uint64_t* stage_free = bars + 19;  // 1 arrival: the copy out of the staging area is done
  uint64_t* xin_read = bars + 20;    // [2] per buffer, 256 arrivals: the peer's partials read
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int n_act_s;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int split = blockIdx.y;
  const int r = blockIdx.x >> 1;
  const int row = p.row_begin + r;
  const int kb_begin = rank == 0 ? 0 : C::VKB;
  const int kb_count = rank == 0 ? C::VKB : C::KBC;
  const int32_t* irow = p.idx + static_cast<int64_t>(r) * p.topk;

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
      mbar_init(smem_u32(&kv_full[i]), 128);
      mbar_init(smem_u32(&kv_empty[i]), 2);
    }
    mbar_init(smem_u32(s_full), 1);
    mbar_init(smem_u32(s_empty), 8);
    mbar_init(smem_u32(p_full), 256);
    mbar_init(smem_u32(pv_done), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&x_full[i]), 1);
      mbar_init(smem_u32(&peer_free[i]), 1);
    }
    mbar_init(smem_u32(mx_bar), 256);
    mbar_init(smem_u32(fin_bar), 256);
    mbar_init(smem_u32(qk_fin), 1);
    mbar_init(smem_u32(pv_fin), 1);
    mbar_init(smem_u32(staged), 256);
    mbar_init(smem_u32(stage_free), 1);
    mbar_init(smem_u32(&xin_read[0]), 256);
    mbar_init(smem_u32(&xin_read[1]), 256);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(&tmem_base_s), C::TMEM_COLS);
  if (warp >= 12) {
    // ---- which tiles hold a valid key (index in [0, n_keys)); warp w takes tiles w, w+4, ..
    const int n_tiles_all = p.topk / C::BN;
    for (int t = warp - 12; t < n_tiles_all; t += 4) {
      const int v0 = irow[t * C::BN + lane], v1 = irow[t * C::BN + 32 + lane];
      if ((v0 >= n_keys || v1 >= n_keys) && p.status) atomicOr(p.status, kStatusBadIndex);
      const uint32_t lo = __ballot_sync(0xffffffffu, v0 >= 0 && v0 < n_keys);
      const uint32_t hi = __ballot_sync(0xffffffffu, v1 >= 0 && v1 < n_keys);
      if (lane == 0) sMask[t] = (static_cast<uint64_t>(hi) << 32) | lo;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  if (warp >= 4 && warp < 12) {
    // ---- this CTA's slice of Q into TMEM (the QK A operand): head = lane, 2 bf16 per column
    const int hrow = (warp & 3) * 32 + lane;
    const int half = (warp - 4) >> 2;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int d0 = kb_begin * 64 + half * kb_count * 32;        // first dim of this half
    const __nv_bfloat16* qrow = p.q + (static_cast<int64_t>(row) * p.h + hrow) * D_QK;
    for (int kb = 0; kb < kb_count; ++kb) {
      uint32_t u[16];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int d = d0 + kb * 32 + c * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (hrow < p.h && d < D_QK) v = *reinterpret_cast<const uint4*>(qrow + d);
        u[4 * c + 0] = v.x;
        u[4 * c + 1] = v.y;
        u[4 * c + 2] = v.z;
        u[4 * c + 3] = v.w;
      }
      tmem_st16(lane_addr + C::Q_COL + half * kb_count * 16 + kb * 16, u);
    }
    tmem_wait_st();
  }
  if (warp == 0 && lane == 0) {
    // ---- the active tiles of this split, identical in both CTAs
    const int n_tiles_all = p.topk / C::BN;
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
    if (t1 - t0 > 0) mbar_arrive_expect_tx(smem_u32(&x_full[0]), C::X_BYTES);   // arm tile 0
    if (t1 - t0 > 1) mbar_arrive_expect_tx(smem_u32(&x_full[1]), C::X_BYTES);   // arm tile 1
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();   // peer barriers initialised before any remote access
  const int n = n_act_s;

  if (warp == 1) {
    // ------------------------------------------------------------ read-signal forwarder
    // Tells the peer, as soon as our softmax has read its partial logits of tile i, that buffer
    // i % 2 may take tile i + 2 (per-buffer barriers: a buffer's reads cannot run two phases
    // ahead of this wait).
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; i < n && ok; ++i) {
        ok = mbar_wait(smem_u32(&xin_read[i & 1]), (i >> 1) & 1, &abort_s);
        if (ok) mbar_arrive_cluster(smem_u32(&peer_free[i & 1]), peer);
      }
      if (!ok) {
        abort_s = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
      }
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ QK issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f32acc(1 /* bf16 */, 128, C::BN, 0, 0);
      bool ok = true;
      for (int i = 0; i < n && ok; ++i) {
        const int s = i % C::STAGES;
        ok = mbar_wait(smem_u32(&kv_full[s]), (i / C::STAGES) & 1, &abort_s);
        if (ok && i >= 1) ok = mbar_wait(smem_u32(s_empty), (i - 1) & 1, &abort_s);
        if (!ok) break;
        tc_fence_after();
        fence_proxy_async_smem();
        const uint32_t ka = smem_u32(sKV + s * C::KV_STAGE_BYTES);
        for (int kb = 0; kb < kb_count; ++kb)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16_ts(tmem + C::S_COL, tmem + C::Q_COL + kb * 32 + k * 8,
                         sdesc_sw128(ka + kb * (C::BN * 128) + k * 32, 16, 1024), idesc,
                         (kb | k) != 0);
        umma_commit(smem_u32(s_full));
        umma_commit(smem_u32(&kv_empty[s]));
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
        const uint32_t va = smem_u32(sKV + s * C::KV_STAGE_BYTES);
#pragma unroll
        for (int k = 0; k < C::BN / 16; ++k)
          umma_bf16_ts(tmem, tmem + C::P_COL + k * 8,
                       sdesc_sw128(va + k * 16 * 128, C::BN * 128, 1024), idesc, (i | k) != 0);
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
  } else if (warp == 3) {
    // ------------------------------------------------------------ exchange copier
    // Copies our staged partial logits of tile i into the peer's buffer (i % 2) once the peer
    // has read tile i - 2 from it; cross-CTA signalling stays off the softmax warps.
    if (lane == 0) {
      const uint32_t xin_remote = map_to_rank(smem_u32(sXin), peer);
      const uint32_t x_full_remote = map_to_rank(smem_u32(x_full), peer);
      bool ok = true;
      for (int i = 0; i < n && ok; ++i) {
        ok = mbar_wait(smem_u32(staged), i & 1, &abort_s);
        if (ok && i >= 2) ok = mbar_wait<true>(smem_u32(&peer_free[i & 1]), ((i >> 1) - 1) & 1,
                                               &abort_s);
        if (!ok) break;
        bulk_copy_to_peer(xin_remote + (i & 1) * C::X_BYTES, smem_u32(sXout), C::X_BYTES,
                          x_full_remote + (i & 1) * 8);
        bulk_commit();
        bulk_wait_read_all();
        mbar_arrive(smem_u32(stage_free));
      }
      if (!ok) {
        abort_s = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
      }
      bulk_wait_read_all();
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ gather producers
    // Producer warp w owns rows [16w, 16w + 16) of every tile: lanes 0..15 resolve their
    // logical key to a physical row (the next tile's index is loaded a tile ahead), then the
    // warp gathers this CTA's dims of its rows with 16-byte cp.async.  No cross-warp barrier.
    const int pw = warp - 12;
    const int chunks = 16 * kb_count * 8;
    int32_t v_next = -1;
    if (n > 0 && lane < 16) v_next = irow[sTiles[0] * C::BN + pw * 16 + lane];
    for (int i = 0; i < n; ++i) {
      const int s = i % C::STAGES;
      if (i >= C::STAGES &&
          !__all_sync(0xffffffffu, mbar_wait(smem_u32(&kv_empty[s]), ((i / C::STAGES) - 1) & 1,
                                             &abort_s))) {
        abort_s = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
        break;
      }
      const int v = v_next;
      if (i + 1 < n && lane < 16) v_next = irow[sTiles[i + 1] * C::BN + pw * 16 + lane];
      int64_t phys = -1;
      if (lane < 16 && v >= 0 && v < n_keys) {
        if (p.decode && p.block_table != nullptr) {
          const int64_t id = __ldg(p.block_table + static_cast<int64_t>(b) * p.max_blocks +
                                   v / p.block_size);
          phys = id < 0 ? -1 : id * p.block_size + v % p.block_size;
        } else {
          phys = key_base + v;
        }
        if (phys >= p.num_kv_rows) phys = -1;
        if (phys < 0 && p.status) atomicOr(p.status, kStatusBadIndex);
      }
      const uint32_t bad = __ballot_sync(0xffffffffu, lane < 16 && v >= 0 && v < n_keys && phys < 0);
      if (lane == 0) sBad[s * 4 + pw] = static_cast<uint16_t>(bad & 0xFFFFu);
      const int32_t my_row = static_cast<int32_t>(phys);
      uint8_t* dst = sKV + s * C::KV_STAGE_BYTES;
      for (int c = lane; c < chunks; c += 32) {
        const int rw = c / (kb_count * 8);          // row within this warp's 16
        const int rem = c % (kb_count * 8);
        const int kbl = rem / 8, ch = rem % 8;
        const int d = (kb_begin + kbl) * 64 + ch * 8;
        const int kr = pw * 16 + rw;                // row within the tile
        const int32_t prow = __shfl_sync(0xffffffffu, my_row, rw);
        const bool ok = prow >= 0 && d < D_QK;
        cp_async_16(smem_u32(dst + kbl * (C::BN * 128) + sw128_offset(kr, ch)),
                    ok ? static_cast<const void*>(p.kv + static_cast<int64_t>(prow) * D_QK + d)
                       : static_cast<const void*>(p.kv),
                    ok ? 16u : 0u);
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&kv_full[s]));
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int quad = warp & 3;
    const int half = (warp - 4) >> 2;           // keys [32 half, 32 half + 32) of each tile
    const int hrow = quad * 32 + lane;          // head = TMEM lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    // row `hrow`, this half, 16-byte chunk c (0..7) of the staged / received partial logits
    const uint32_t x_row = half * (128 * 128) + hrow * 128;
    constexpr int OC = C::V_HALF / 2;           // O columns this half rescales / stores
    float m_ref = -INFINITY, l_sum = 0.f;
    float own[32];                              // our partial logits of the tile in flight
    bool ok = true;
    // Loads S(j) from TMEM, frees it for the next QK, stages it for the peer; keeps our partial.
    auto stage_tile = [&](int j) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(s_full), j & 1, &abort_s))) return false;
      tc_fence_after();
      uint32_t u[32];
      tmem_ld32(lane_addr + C::S_COL + half * 32, u);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) own[e] = __uint_as_float(u[e]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(s_empty));
      if (j >= 1 &&
          !__all_sync(0xffffffffu, mbar_wait(smem_u32(stage_free), (j - 1) & 1, &abort_s)))
        return false;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<float4*>(sXout + x_row + ((c ^ (hrow & 7)) << 4)) =
            make_float4(own[4 * c], own[4 * c + 1], own[4 * c + 2], own[4 * c + 3]);
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(staged));
      return true;
    };
    if (n > 0) ok = stage_tile(0);
    for (int i = 0; i < n && ok; ++i) {
      float sv[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) sv[e] = own[e];
      // start the swap of the next tile before working on this one
      if (i + 1 < n) {
        ok = stage_tile(i + 1);
        if (!ok) break;
      }
      const int xb = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait<true>(smem_u32(&x_full[xb]), (i >> 1) & 1, &abort_s));
      if (!ok) break;
      if (warp == 4 && lane == 0 && i + 2 < n)
        mbar_arrive_expect_tx(smem_u32(&x_full[xb]), C::X_BYTES);   // arm tile i+2
      // the producers' invalid-row bits of this tile: observe its kv_full phase first (the
      // stage is not refilled before PV(i), which needs this tile's P)
      const int st = i % C::STAGES;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&kv_full[st]), (i / C::STAGES) & 1, &abort_s));
      if (!ok) break;
      const uint64_t bad = static_cast<uint64_t>(sBad[st * 4 + 0]) |
                           (static_cast<uint64_t>(sBad[st * 4 + 1]) << 16) |
                           (static_cast<uint64_t>(sBad[st * 4 + 2]) << 32) |
                           (static_cast<uint64_t>(sBad[st * 4 + 3]) << 48);
      const uint64_t vmask = sMask[sTiles[i]] & ~bad;
      const uint32_t vbits = static_cast<uint32_t>(vmask >> (32 * half));
      const uint8_t* xin = sXin + xb * C::X_BYTES;
      float m_half = -INFINITY;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 o = *reinterpret_cast<const float4*>(xin + x_row + ((c ^ (hrow & 7)) << 4));
        const float ov[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 4 * c + e;
          // both CTAs add rank 0's partial to rank 1's: bit-identical logits in both
          const float full_s = rank == 0 ? sv[j] + ov[e] : ov[e] + sv[j];
          sv[j] = ((vbits >> j) & 1u) ? full_s * p.scale_log2 : -INFINITY;
          m_half = fmaxf(m_half, sv[j]);
        }
      }
      mbar_arrive(smem_u32(&xin_read[xb]));
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
           rank * C::V_HALF;
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
        __nv_bfloat16* dst = p.out + orow * D_V + rank * C::V_HALF + c0;
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
    if (write && rank == 0 && half == 0) {
      if (p.part_lse != nullptr)
        p.part_lse[(static_cast<int64_t>(split) * p.row_count + r) * p.h + hrow] = lse_v;
      else
        p.lse[orow] = lse_v;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // no remote access to this CTA's shared memory after this point
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
