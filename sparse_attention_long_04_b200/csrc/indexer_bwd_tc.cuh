// Backward of the lightning indexer against its KL training target, on the tensor cores
// (indexer shape 64 heads x 128 dims).  It computes what the CUDA-core kernel in indexer_bwd.cuh
// computes ("DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek Sparse Attention (DSA)",
// "Training signal"; the formulas are stated there), with the three contractions of each row
// as tcgen05 MMAs over 128-key tiles of its selection:
//   D^T = Kh Qh^T        e4m3, M = 128 keys, N = 64 heads, K = 128 dims (the indexer's shape)
//   dk  = g (M1 Qw)      bf16, M = 128 keys, N = 128 dims, K = 2 x 64 heads;
//                        M1[e][j] = [D_je > 0] (exact 0/1), Qw[j][d] = w_j s_q,j Qh[j][d] as a
//                        bf16 pair hi + lo stacked along K; g_e applied in fp32 afterwards
//   dq  += B2^T Kh       bf16, M = 2 x 64 heads (hi rows, then lo rows), N = 128 dims,
//                        K = 128 keys; B2[e][j] = g_e s_k,e [D_je > 0] as a pair hi + lo;
//                        the two halves are added once at the end
// Qh and Kh (e4m3 codes) are exact in bf16; a coefficient split into hi = bf16(x) and
// lo = bf16(x - hi) keeps 16 significant bits, so the gradients stay at fp32-accumulation
// accuracy even where g cancels.
//
// One CTA per query row (1 per SM: it allocates all 512 TMEM columns).  Warp 0 issues the MMAs,
// warp 1 owns TMEM, warps 2-3 gather each tile (16-byte cp.async of the selected key rows into
// a 128-byte-swizzled tile and of the tile's targets, 4-byte copies of the keys' scales; 8
// stages in pass 1, 2 in pass 2; unused entries read as zeros), warps 4-7 are the epilogue with
// thread = TMEM lane.
// Pass 1 runs D^T for every tile (4 accumulators in rotation, so the MMAs run ahead of the
// epilogue) and the epilogue forms the scores S (thread = key), keeping per thread the running
// softmax statistics of its keys (max, the sum of exp(S - max), and the target's sum, sum p S
// and sum p ln p); the 128 epilogue threads then combine them into the normaliser and the loss.
// No per-key value is stored, so a row may have any number of entries.  When the selected keys'
// scores are given (the forward's top-k keeps them), pass 1 reads them instead, with no gather
// and no MMA, and pass 2 takes S from them too.  Pass 2 runs D^T again per tile, recomputes S
// with the same instructions (so the same value and ReLU decisions) and forms g; the epilogue sums dw over the tile's keys with a butterfly across lanes and writes
// M1 (TMEM, thread = key), B2 and the key tile in bf16 (shared memory, row = key).  The dk
// accumulator is double-buffered: while the tensor cores run tile i's dk and dq, the epilogue
// drains tile i-1's dk rows (times g) through shared memory into global memory with bulk
// reductions (one 512-byte cp.reduce.async.bulk per key), then forms tile i+1's operands.  At
// the end the epilogue writes dq (hi + lo, times w) and dw.  Every wait is bounded.
//
// Dense mode (the warm-up stage of the training, "Training signal": the indexer imitates the
// dense attention over every prior key): no index array; the entries of row t are its keys
// 0..pos(t) (prefill: consecutive packed rows), in 128-key tiles computed on the fly, and the
// target row has one entry per key.
#pragma once
#include <cuda_bf16.h>

#include "indexer_bwd.cuh"
#include "sm100.cuh"

namespace dsa {

struct KlTcCfg {
  static constexpr int H = 64, D = 128;            // indexer heads and dims
  static constexpr int BK = 128;                   // keys per tile (MMA M of D^T and dk)
  static constexpr int MAX_K = 2048;
  static constexpr int MAX_TILES = MAX_K / BK;
  static constexpr int STAGES = 2;                 // key stages of pass 2
  static constexpr int STAGES1 = 8;                // key stages of pass 1: the 2 above and 6
                                                   // over the pass-2 buffers B2 and staging
  static constexpr int ND1 = 4;                    // D^T buffers of pass 1 (over dk, dq)
  static constexpr int THREADS = 256;
  static constexpr int TILE_BYTES = BK * D;        // e4m3 key rows, 16 KB
  static constexpr int BF_TILE = 2 * BK * 128;     // bf16 [2 blocks of 64][128 rows][128 B]
  static constexpr int STAGE_ROW = D * 4 + 16;     // dk staging row (padded: no bank conflicts)
  // Tensor Memory columns
  static constexpr int D_COL = 0;                  // D^T [128 keys x 64 heads] fp32
  static constexpr int DK_COL = 64;                // dk tiles [128 keys x 128 dims] fp32, x 2
  static constexpr int DQ_COL = 320;               // dq [2 x 64 heads x 128 dims] fp32 (row)
  static constexpr int M1_COL = 448;               // M1 [128 keys x 2 x 64 heads]: bf16 pairs
  static constexpr int TMEM_COLS = 512;
  // shared memory, from a 1024-byte-aligned base
  static constexpr int OFF_Q8 = 0;                             // [64 heads][128 B] e4m3 K-major
  static constexpr int OFF_QW = OFF_Q8 + H * D;                // Qw hi/lo, MN-major bf16
  static constexpr int OFF_KT = OFF_QW + BF_TILE;              // [STAGES][128 keys][128 B] e4m3
  static constexpr int OFF_KH = OFF_KT + STAGES * TILE_BYTES;  // key tile in bf16, MN-major
  static constexpr int OFF_B2 = OFF_KH + BF_TILE;              // B2 hi/lo, MN-major bf16
  static constexpr int OFF_STG = OFF_B2 + BF_TILE;             // [128 keys][STAGE_ROW] dk rows
  static constexpr int OFF_KS = OFF_STG + BK * STAGE_ROW;      // [STAGES1][128] k_scale
  static constexpr int OFF_TG = OFF_KS + STAGES1 * BK * 4;     // [STAGES1][128] target
  static constexpr int OFF_PHYS = OFF_TG + STAGES1 * BK * 4;   // [MAX_K] i32 (selected keys)
  static constexpr int OFF_TILES = OFF_PHYS + 4 * MAX_K;       // [MAX_TILES] i32
  static constexpr int OFF_W = OFF_TILES + 4 * MAX_TILES;      // [64] w
  static constexpr int OFF_SQ = OFF_W + 4 * H;                 // [64] s_q
  static constexpr int OFF_DWP = OFF_SQ + 4 * H;               // [4 warps][64] dw partials
  static constexpr int OFF_SCR = OFF_DWP + 4 * 4 * H;          // [32] reduction scratch
  static constexpr int OFF_BAR = OFF_SCR + 4 * 32;             // barriers
  static constexpr int N_BAR = 2 * STAGES1 + 2 * ND1 + 8;
  static constexpr int USED = OFF_BAR + 8 * N_BAR;
  static constexpr int SMEM_BYTES = 1024 + USED;
  static_assert(OFF_QW % 1024 == 0 && OFF_KT % 1024 == 0 && OFF_KH % 1024 == 0 &&
                OFF_B2 % 1024 == 0, "tiles");
  static_assert(OFF_STG % 16 == 0 && STAGE_ROW % 16 == 0, "bulk sources");
  static_assert(OFF_BAR % 8 == 0, "barriers");
  static_assert((STAGES1 - STAGES) * TILE_BYTES <= BF_TILE + BK * STAGE_ROW &&
                    OFF_STG == OFF_B2 + BF_TILE,
                "pass-1 stages over B2 and the staging rows");
  static_assert(D_COL == 0 && (ND1 - 1) * 64 <= DQ_COL - DK_COL + 64, "pass-1 D^T buffers");
  // key stage of step `it` (pass 1: it < n; pass 2: it = n + i) and how often that stage was
  // used before it (the parity of its barriers); n1 = the pass-1 steps that ran on the keys
  // (n, or 0 when the scores are given)
  __device__ static int stage_of(int it, int n) {
    return it < n ? it % STAGES1 : (it - n) % STAGES;
  }
  __device__ static int use_of(int it, int n, int n1) {
    if (it < n) return it / STAGES1;
    const int s = (it - n) % STAGES;
    const int used1 = n1 > s ? (n1 - 1 - s) / STAGES1 + 1 : 0;
    return used1 + (it - n) / STAGES;
  }
  // D^T buffer of step `it` (pass 1 rotates over ND1 buffers at columns 64 b; pass 2 uses
  // buffer 0) and how often that buffer was used before it
  __device__ static int dbuf_of(int it, int n) { return it < n ? it % ND1 : 0; }
  __device__ static int duse_of(int it, int n, int n1) {
    return it < n ? it / ND1 : (n1 + ND1 - 1) / ND1 + (it - n);
  }
  static_assert(SMEM_BYTES > 116 * 1024, "one CTA per SM (its TMEM allocation never waits)");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// bf16 pair (a in the low half) as one 32-bit word
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&t);
}

// x = hi + lo with hi = bf16(x), lo = bf16(x - hi); returns the two packed pairs of (x0, x1)
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = pack_bf16(x0 - hf.x, x1 - hf.y);
}

// two e4m3 codes (low byte first) as a bf16 pair, exactly
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two) {
  const __half2 hv = __half2(__nv_cvt_fp8x2_to_halfraw2(
      static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu), __NV_E4M3));
  const float2 f = __half22float2(hv);
  return pack_bf16(f.x, f.y);
}

__global__ void __launch_bounds__(256, 1) dsa_indexer_kl_bwd_tc_kernel(const IdxBwdParams p) {
  using C = KlTcCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ8 = smem + C::OFF_Q8;
  uint8_t* sQw = smem + C::OFF_QW;
  uint8_t* sKt = smem + C::OFF_KT;
  uint8_t* sKh = smem + C::OFF_KH;
  uint8_t* sB2 = smem + C::OFF_B2;
  uint8_t* sStg = smem + C::OFF_STG;
  float* sKs = reinterpret_cast<float*>(smem + C::OFF_KS);
  float* sTg = reinterpret_cast<float*>(smem + C::OFF_TG);
  int32_t* sPhys = reinterpret_cast<int32_t*>(smem + C::OFF_PHYS);
  int32_t* sTiles = reinterpret_cast<int32_t*>(smem + C::OFF_TILES);
  float* sW = reinterpret_cast<float*>(smem + C::OFF_W);
  float* sSq = reinterpret_cast<float*>(smem + C::OFF_SQ);
  float* sDwp = reinterpret_cast<float*>(smem + C::OFF_DWP);
  float* sScr = reinterpret_cast<float*>(smem + C::OFF_SCR);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;            // [STAGES1] 64 gathering threads (each when its copies land)
  uint64_t* kempty = full + C::STAGES1;   // [STAGES1] 128 epilogue threads: stage no longer read
  uint64_t* d_full = kempty + C::STAGES1;   // [ND1] D^T MMA commit
  uint64_t* d_empty = d_full + C::ND1;      // [ND1] 128 epilogue threads: D^T read
  uint64_t* coef_full = d_empty + C::ND1;   // 128 epilogue threads: M1, B2, Kh written (and
                                            // the dk buffer of two tiles back drained)
  uint64_t* mma_done = coef_full + 1;  // dk / dq MMA commit
  uint64_t* ep_bar = coef_full + 2;    // 128 epilogue threads meet
  uint64_t* fin = coef_full + 3;       // the MMA issuer's last commit
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int n_act_s;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int r = blockIdx.x;
  const int row = p.row_begin + r;
  const bool dense = p.dense != 0;

  // ---- row geometry
  int b, n_keys;
  int64_t key_base = 0;
  if (p.decode) {
    b = row;
    n_keys = min(p.seq_lens[b], p.max_seqlen);
    key_base = static_cast<int64_t>(b) * p.kv_stride;
  } else {
    int lo = 0, hi = p.batch;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.cu_seqlens[mid] <= row) lo = mid; else hi = mid;
    }
    b = lo;
    n_keys = row - p.cu_seqlens[lo] + 1;
    key_base = p.cu_seqlens[lo];
  }

  // ---- prologue: queries (e4m3 K-major for D^T), w, s_q, Qw (hi/lo MN-major for dk), keys
  const uint8_t* qrow = p.q_idx + static_cast<int64_t>(row) * C::H * C::D;
  for (int u = tid; u < C::H * 8; u += C::THREADS) {
    const int j = u >> 3, c = u & 7;
    *reinterpret_cast<uint4*>(sQ8 + sw128_offset(j, c)) =
        __ldg(reinterpret_cast<const uint4*>(qrow + j * C::D + c * 16));
  }
  if (tid < C::H) {
    sW[tid] = __ldg(p.w + static_cast<int64_t>(row) * C::H + tid);
    sSq[tid] = __ldg(p.q_scale + static_cast<int64_t>(row) * C::H + tid);
  }
  __syncthreads();
  for (int u = tid; u < C::H * 16; u += C::THREADS) {
    const int j = u >> 4, dc = u & 15;             // head j, dims [8 dc, 8 dc + 8)
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(qrow + j * C::D + dc * 8));
    const float cj = sW[j] * sSq[j];
    const float4 f0 = decode4_e4m3(raw.x, cj), f1 = decode4_e4m3(raw.y, cj);
    uint32_t hw[4], lw[4];
    split_bf16(f0.x, f0.y, hw[0], lw[0]);
    split_bf16(f0.z, f0.w, hw[1], lw[1]);
    split_bf16(f1.x, f1.y, hw[2], lw[2]);
    split_bf16(f1.z, f1.w, hw[3], lw[3]);
    uint8_t* blk = sQw + (dc >> 3) * (2 * C::H * 128);
    *reinterpret_cast<uint4*>(blk + sw128_offset(j, dc & 7)) =
        make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(blk + sw128_offset(C::H + j, dc & 7)) =
        make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
  const int K = dense ? n_keys : p.topk;   // entries of the row
  if (!dense) {
    bool bad = false;
    const int32_t* irow = p.idx + static_cast<int64_t>(r) * K;
    for (int e = tid; e < K; e += C::THREADS) {
      const int v = __ldg(irow + e);
      int64_t ph = -1;
      if (v >= n_keys) bad = true;
      if (v >= 0 && v < n_keys) {
        if (p.decode && p.block_table != nullptr) {
          const int32_t blk =
              __ldg(p.block_table + static_cast<int64_t>(b) * p.max_blocks + v / p.block_size);
          ph = blk < 0 ? -1 : static_cast<int64_t>(blk) * p.block_size + v % p.block_size;
        } else {
          ph = key_base + v;
        }
        if (ph >= p.num_kv_rows) ph = -1;
        if (ph < 0) bad = true;
      }
      sPhys[e] = static_cast<int32_t>(ph);
    }
    if (bad && p.status) atomicOr(p.status, kStatusBadIndex);
  }
  if (tid == 0) {
    for (int i = 0; i < C::STAGES1; ++i) {
      mbar_init(smem_u32(&full[i]), 64);
      mbar_init(smem_u32(&kempty[i]), 128);
    }
    for (int i = 0; i < C::ND1; ++i) {
      mbar_init(smem_u32(&d_full[i]), 1);
      mbar_init(smem_u32(&d_empty[i]), 128);
    }
    mbar_init(smem_u32(coef_full), 128);
    mbar_init(smem_u32(mma_done), 1);
    mbar_init(smem_u32(ep_bar), 128);
    mbar_init(smem_u32(fin), 1);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(&tmem_base_s), C::TMEM_COLS);
  fence_proxy_async_smem();   // the query tiles are read by the tensor cores
  __syncthreads();
  if (tid == 0) {
    int n = 0;
    if (dense) {
      n = (n_keys + C::BK - 1) / C::BK;
    } else {
      for (int t = 0; t < K / C::BK; ++t) {
        bool any = false;
        for (int e = 0; e < C::BK && !any; ++e) any = sPhys[t * C::BK + e] >= 0;
        if (any) sTiles[n++] = t;
      }
    }
    n_act_s = n;
  }
  // tile of step i and physical row of entry e (-1: unused entry)
  auto tile_at = [&](int i) -> int { return dense ? i : sTiles[i]; };
  auto phys_at = [&](int e) -> int64_t {
    if (!dense) return sPhys[e];
    return e < n_keys ? key_base + e : -1;
  };
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const int n = n_act_s;
  const int steps = 2 * n;   // pass 1 then pass 2 over the same tiles
  // with the selected keys' scores given, pass 1 reads them instead of the keys: the gather and
  // the MMAs start at pass 2
  const bool have_sel = p.sel != nullptr && !dense;
  const int n1 = have_sel ? 0 : n;
  const int it0 = n - n1;
  const float* selrow = have_sel ? p.sel + static_cast<int64_t>(r) * K : nullptr;
  // e4m3 key tile of stage s (stages 2.. lie over B2 and the staging rows, which only the
  // epilogue writes, in pass 2, after every pass-1 MMA has completed)
  auto key_tile = [&](int s) -> uint8_t* {
    return s < C::STAGES ? sKt + s * C::TILE_BYTES : sB2 + (s - C::STAGES) * C::TILE_BYTES;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ MMA issuer
    // Step it issues D^T of step it, then (pass 2) dk and dq of the tile before it, so that the
    // next tile's scores are on their way while the epilogue forms this tile's operands.
    if (lane == 0) {
      constexpr uint32_t id_d = idesc_f32acc(0 /* e4m3 */, 128, 64, 0, 0);
      constexpr uint32_t id_dk = idesc_f32acc(1 /* bf16 */, 128, 128, 0, 1);
      constexpr uint32_t id_dq = idesc_f32acc(1 /* bf16 */, 128, 128, 1, 1);
      const uint32_t q8 = smem_u32(sQ8), qw = smem_u32(sQw), b2 = smem_u32(sB2),
                     kh = smem_u32(sKh);
      bool ok = true;
      for (int it = it0; it <= steps && ok; ++it) {
        if (it < steps) {
          const int s = C::stage_of(it, n);
          const int db = C::dbuf_of(it, n), du = C::duse_of(it, n, n1);
          ok = mbar_wait(smem_u32(&full[s]), C::use_of(it, n, n1) & 1, &abort_s);
          if (ok && du >= 1) ok = mbar_wait(smem_u32(&d_empty[db]), (du - 1) & 1, &abort_s);
          if (!ok) break;
          tc_fence_after();
          fence_proxy_async_smem();   // the key tile was written by cp.async
          const uint32_t kt = smem_u32(key_tile(s));
#pragma unroll
          for (int k = 0; k < C::D / 32; ++k)
            umma_e4m3(tmem + C::D_COL + 64 * db, sdesc_sw128(kt + k * 32, 16, 1024),
                      sdesc_sw128(q8 + k * 32, 16, 1024), id_d, k > 0);
          umma_commit(smem_u32(&d_full[db]));
        }
        const int i2 = it - 1 - n;   // pass-2 tile whose dk and dq run now
        if (i2 < 0) continue;
        ok = mbar_wait(smem_u32(coef_full), i2 & 1, &abort_s);
        if (!ok) break;
        tc_fence_after();
        fence_proxy_async_smem();   // B2 and Kh were written with st.shared
        const uint32_t dk_col = tmem + C::DK_COL + 128 * (i2 & 1);
#pragma unroll
        for (int k = 0; k < 2 * C::H / 16; ++k)
          umma_bf16_ts(dk_col, tmem + C::M1_COL + 8 * k,
                       sdesc_sw128(qw + k * 16 * 128, 2 * C::H * 128, 1024), id_dk, k != 0);
#pragma unroll
        for (int k = 0; k < C::BK / 16; ++k)
          umma_bf16(tmem + C::DQ_COL, sdesc_sw128(b2 + k * 16 * 128, C::BK * 128, 1024),
                    sdesc_sw128(kh + k * 16 * 128, C::BK * 128, 1024), id_dq, (i2 | k) != 0);
        umma_commit(smem_u32(mma_done));
      }
      if (!ok) {
        abort_s = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
      }
      umma_commit(smem_u32(fin));
      mbar_wait(smem_u32(fin), 0, nullptr);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ gather
    // thread pt copies 16-byte chunk (pt & 7) of rows (pt >> 3) + 8 q of every tile, the scales
    // of entries pt and pt + 64 (4 bytes each) and, pt < 32, 16-byte chunk pt of the targets
    const int pt = tid - 64;
    const int c = pt & 7, r0 = pt >> 3;
    const float* trow = p.target + static_cast<int64_t>(r) * p.ld_target;
    bool ok = true;
    for (int it = it0; it < steps && ok; ++it) {
      const int s = C::stage_of(it, n), u = C::use_of(it, n, n1);
      if (u >= 1 && !warp_mbar_wait(smem_u32(&kempty[s]), (u - 1) & 1, &abort_s)) {
        ok = false;
        break;
      }
      const int tile = tile_at(it % n);
      const uint32_t dst = smem_u32(key_tile(s));
#pragma unroll 4
      for (int q = 0; q < C::BK / 8; ++q) {
        const int rr = r0 + 8 * q;
        const int64_t ph = phys_at(tile * C::BK + rr);
        const void* src = ph >= 0 ? static_cast<const void*>(p.k_idx + static_cast<int64_t>(ph) *
                                                                         C::D + c * 16)
                                  : static_cast<const void*>(p.k_idx);
        cp_async_16(dst + sw128_offset(rr, c), src, ph >= 0 ? 16u : 0u);   // unused: zeros
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int ee = pt + 64 * q;
        const int64_t ph = phys_at(tile * C::BK + ee);
        cp_async_4(smem_u32(sKs + s * C::BK + ee), ph >= 0 ? p.k_scale + ph : p.k_scale,
                   ph >= 0 ? 4u : 0u);
      }
      if (pt < C::BK / 4) {
        // targets [tile 128 + 4 pt, +4): within the row's stride (a multiple of 4), else zeros
        const int64_t e4 = static_cast<int64_t>(tile) * C::BK + 4 * pt;
        const bool in = e4 < p.ld_target;
        cp_async_16(smem_u32(sTg + s * C::BK + 4 * pt), in ? trow + e4 : trow, in ? 16u : 0u);
      }
      cp_async_arrive_noinc(smem_u32(&full[s]));
    }
    if (!ok) {
      abort_s = 1;
      if (p.status) atomicOr(p.status, kStatusTimeout);
    }
    cp_async_wait_all();   // nothing may still be writing this CTA's shared memory at exit
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue (thread = TMEM lane)
    const int et = tid - 128, ew = et >> 5;
    const uint32_t la = tmem + (static_cast<uint32_t>(ew * 32) << 16);
    int ep_phase = 0;
    auto epi_sync = [&]() -> bool {
      mbar_arrive(smem_u32(ep_bar));
      const bool r2 = warp_mbar_wait(smem_u32(ep_bar), ep_phase & 1, &abort_s);
      ++ep_phase;
      return r2;
    };
    bool ok = true;
    // ---- pass 1: S_e = s_k sum_j w_j s_q,j max(D_je, 0), thread = key; running statistics
    // (explicitly rounded products: pass 2 must get the bits of pass 1, so the compiler may not
    // fuse them into the arithmetic that follows either call)
    auto score = [&](const uint32_t (&du)[2][32], float ks) -> float {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < C::H; ++j)
        acc = fmaf(__fmul_rn(sW[j], sSq[j]), fmaxf(__uint_as_float(du[j >> 5][j & 31]), 0.f),
                   acc);
      return __fmul_rn(ks, acc);
    };
    // this step's D^T, its scale and target (the stage's barrier, already complete, orders the
    // cp.async data before the shared-memory reads)
    auto read_step = [&](int it, uint32_t (&du)[2][32], float& ks, float& tg) -> bool {
      const int s = C::stage_of(it, n);
      const int db = C::dbuf_of(it, n);
      if (!warp_mbar_wait(smem_u32(&d_full[db]), C::duse_of(it, n, n1) & 1, &abort_s))
        return false;
      tc_fence_after();
      tmem_ld32(la + C::D_COL + 64 * db, du[0]);
      tmem_ld32(la + C::D_COL + 64 * db + 32, du[1]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(&d_empty[db]));
      if (!warp_mbar_wait(smem_u32(&full[s]), C::use_of(it, n, n1) & 1, &abort_s)) return false;
      ks = sKs[s * C::BK + et];
      tg = sTg[s * C::BK + et];
      return true;
    };
    float m = -INFINITY, z = 0.f, psum = 0.f, sps = 0.f, splp = 0.f;
    auto stats = [&](float S, float pe) {
      if (S > m) {
        z = z * expf(m - S) + 1.f;
        m = S;
      } else {
        z += expf(S - m);
      }
      psum += pe;
      sps += pe * S;
      if (pe > 0.f) splp += pe * logf(pe);
    };
    if (have_sel) {
      // the scores and targets of this thread's entries, straight from global memory
      const float* trow = p.target + static_cast<int64_t>(r) * p.ld_target;
      for (int it = 0; it < n; it += 4) {
        float sv[4], pv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = it + u < n ? tile_at(it + u) * C::BK + et : -1;
          sv[u] = e >= 0 && phys_at(e) >= 0 ? __ldg(selrow + e) : 0.f;
          pv[u] = e >= 0 && phys_at(e) >= 0 ? __ldg(trow + e) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (it + u < n && phys_at(tile_at(it + u) * C::BK + et) >= 0) stats(sv[u], pv[u]);
      }
    }
    for (int it = 0; it < n1 && ok; ++it) {
      uint32_t du[2][32];
      float ks, pe;
      ok = read_step(it, du, ks, pe);
      if (!ok) break;
      mbar_arrive(smem_u32(&kempty[C::stage_of(it, n)]));
      if (phys_at(tile_at(it) * C::BK + et) >= 0) stats(score(du, ks), pe);
    }
    // ---- the row's normaliser and loss from the 128 threads' statistics
    const float wm = warp_max(m);
    float zz = m == -INFINITY ? 0.f : z * expf(m - wm);
    zz = warp_sum(zz);
    psum = warp_sum(psum);
    sps = warp_sum(sps);
    splp = warp_sum(splp);
    if (lane == 0) {
      sScr[ew] = wm;
      sScr[4 + ew] = zz;
      sScr[8 + ew] = psum;
      sScr[12 + ew] = sps;
      sScr[16 + ew] = splp;
    }
    ok = ok && epi_sync();
    m = fmaxf(fmaxf(sScr[0], sScr[1]), fmaxf(sScr[2], sScr[3]));
    z = 0.f;
#pragma unroll
    for (int w4 = 0; w4 < 4; ++w4)
      if (sScr[w4] != -INFINITY) z += sScr[4 + w4] * expf(sScr[w4] - m);
    psum = (sScr[8] + sScr[9]) + (sScr[10] + sScr[11]);
    sps = (sScr[12] + sScr[13]) + (sScr[14] + sScr[15]);
    splp = (sScr[16] + sScr[17]) + (sScr[18] + sScr[19]);
    const float log_z = m == -INFINITY ? 0.f : m + logf(z);
    // loss = sum p (ln p - ln pi), ln pi = S - log_z
    if (et == 0) p.loss[r] = (m == -INFINITY || !ok) ? 0.f : splp - sps + psum * log_z;

    // ---- pass 2
    // dk rows of the tile in buffer `buf`, times g, into this thread's staging row, then added
    // to global memory by the bulk engine
    uint8_t* my_stage = sStg + et * C::STAGE_ROW;
    auto drain = [&](int buf, float g, int64_t ph) {
      bulk_wait_read_all();   // the previous reduction has read this staging row
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {   // 64 columns per wait
        uint32_t u[2][32];
        tmem_ld32(la + C::DK_COL + 128 * buf + 64 * hh, u[0]);
        tmem_ld32(la + C::DK_COL + 128 * buf + 64 * hh + 32, u[1]);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4)
            *reinterpret_cast<float4*>(my_stage + 256 * hh + 128 * q + 16 * c4) =
                make_float4(g * __uint_as_float(u[q][4 * c4]), g * __uint_as_float(u[q][4 * c4 + 1]),
                            g * __uint_as_float(u[q][4 * c4 + 2]),
                            g * __uint_as_float(u[q][4 * c4 + 3]));
      }
      fence_proxy_async_smem();   // the staging row is read by the bulk engine
      if (ph >= 0 && g != 0.f) {
        bulk_reduce_add_f32(p.dk + ph * C::D, smem_u32(my_stage), C::D * 4);
        bulk_commit();
      }
    };
    const int h0 = warp_sum64_first(lane);   // this lane's two heads of the warp's dw sums
    float dw0 = 0.f, dw1 = 0.f;
    float g_prev = 0.f;
    int64_t ph_prev = -1;
    for (int i2 = 0; i2 < n && ok; ++i2) {
      const int it = n + i2, s = C::stage_of(it, n);
      const int e2 = tile_at(i2) * C::BK + et;
      const int64_t ph = phys_at(e2);
      const float s_given = have_sel && ph >= 0 ? __ldg(selrow + e2) : 0.f;
      uint32_t du[2][32];
      float ks, tg;
      ok = read_step(it, du, ks, tg);
      if (!ok) break;
      // g = pi psum - p, from the same score as in pass 1 (0 for unused entries)
      const float g = ph >= 0 ? expf((have_sel ? s_given : score(du, ks)) - log_z) * psum - tg
                              : 0.f;
      const float gsk = g * ks;
      // dw: g s_k max(D, 0) summed over the tile's keys (s_q applied at the end)
      {
        float v[64];
#pragma unroll
        for (int j = 0; j < C::H; ++j) v[j] = gsk * fmaxf(__uint_as_float(du[j >> 5][j & 31]), 0.f);
        warp_sum64(v, lane);
        dw0 += v[0];
        dw1 += v[1];
      }
      // the previous tile's dk and dq are done: M1, B2 and Kh may be overwritten
      if (i2 >= 1) {
        ok = warp_mbar_wait(smem_u32(mma_done), (i2 - 1) & 1, &abort_s);
        if (!ok) break;
        tc_fence_after();
      }
      // M1 = [D > 0] (1.0 / 0.0 in bf16), twice along K (for Qw hi and lo), this key's lane
      {
        uint32_t mw[32];
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) {
          const int j = 2 * c2;
          mw[c2] = (__uint_as_float(du[j >> 5][j & 31]) > 0.f ? 0x3F80u : 0u) |
                   (__uint_as_float(du[(j + 1) >> 5][(j + 1) & 31]) > 0.f ? 0x3F800000u : 0u);
        }
        tmem_st32(la + C::M1_COL, mw);
        tmem_st32(la + C::M1_COL + 32, mw);
      }
      // B2 = g s_k [D > 0] (hi, lo): row et of the hi block and of the lo block
      {
        uint32_t ghi, glo;
        split_bf16(gsk, gsk, ghi, glo);
        const uint32_t hh = ghi & 0xFFFFu, ll = glo & 0xFFFFu;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int j = 8 * c8 + 2 * q;
            const bool a0 = __uint_as_float(du[j >> 5][j & 31]) > 0.f;
            const bool a1 = __uint_as_float(du[(j + 1) >> 5][(j + 1) & 31]) > 0.f;
            hw[q] = (a0 ? hh : 0u) | (a1 ? hh << 16 : 0u);
            lw[q] = (a0 ? ll : 0u) | (a1 ? ll << 16 : 0u);
          }
          *reinterpret_cast<uint4*>(sB2 + sw128_offset(et, c8)) =
              make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(sB2 + C::BK * 128 + sw128_offset(et, c8)) =
              make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      }
      // Kh: this thread's key row of the tile in bf16 (exact), row et of the two dim blocks
      {
        const uint8_t* tb = key_tile(s);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(tb + sw128_offset(et, c));
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
          uint32_t o[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            o[2 * q] = e4m3x2_to_bf16x2(wv[q]);
            o[2 * q + 1] = e4m3x2_to_bf16x2(wv[q] >> 16);
          }
          uint8_t* blk = sKh + (c >> 2) * (C::BK * 128);
          *reinterpret_cast<uint4*>(blk + sw128_offset(et, 2 * (c & 3))) =
              make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(blk + sw128_offset(et, 2 * (c & 3) + 1)) =
              make_uint4(o[4], o[5], o[6], o[7]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();   // B2 and Kh are read by the tensor cores
      tc_fence_before();
      mbar_arrive(smem_u32(&kempty[s]));
      mbar_arrive(smem_u32(coef_full));
      // the previous tile's dk, while this tile's runs
      if (i2 >= 1) drain((i2 - 1) & 1, g_prev, ph_prev);
      g_prev = g;
      ph_prev = ph;
    }
    if (ok && n > 0) {
      ok = warp_mbar_wait(smem_u32(mma_done), (n - 1) & 1, &abort_s);
      if (ok) {
        tc_fence_after();
        drain((n - 1) & 1, g_prev, ph_prev);
      }
    }
    bulk_wait_all();   // every reduction done: the staging rows are free, dk is written
    if (!ok) {
      abort_s = 1;
      if (p.status) atomicOr(p.status, kStatusTimeout);
    }
    // ---- dw: the four warps' partial sums, times s_q
    sDwp[ew * C::H + h0] = dw0;
    sDwp[ew * C::H + h0 + 1] = dw1;
    const bool met = ok && epi_sync();
    if (et < C::H)
      p.dw[static_cast<int64_t>(r) * C::H + et] =
          met ? ((sDwp[et] + sDwp[C::H + et]) + (sDwp[2 * C::H + et] + sDwp[3 * C::H + et])) *
                    sSq[et]
              : 0.f;
    // ---- dq[j][d] = w_j (hi[j][d] + lo[j][d]): lanes 64..127 (lo) pass their rows through
    // the staging area to lanes 0..63 (hi), which write the head rows
    if (ew >= 2) {
#pragma unroll
      for (int q = 0; q < C::D / 32; ++q) {
        uint32_t u[32];
        tmem_ld32(la + C::DQ_COL + 32 * q, u);
        tmem_wait_ld();
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4)
          *reinterpret_cast<uint4*>(my_stage + 128 * q + 16 * c4) =
              make_uint4(u[4 * c4], u[4 * c4 + 1], u[4 * c4 + 2], u[4 * c4 + 3]);
      }
    }
    const bool met2 = met && epi_sync();
    if (ew < 2) {
      const uint8_t* lo_row = sStg + (et + C::H) * C::STAGE_ROW;
      float4* dq = reinterpret_cast<float4*>(p.dq + (static_cast<int64_t>(r) * C::H + et) * C::D);
      const float wj = sW[et];
      const bool good = met2 && n > 0;
#pragma unroll
      for (int q = 0; q < C::D / 32; ++q) {
        uint32_t u[32];
        tmem_ld32(la + C::DQ_COL + 32 * q, u);
        tmem_wait_ld();
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lo_row + 128 * q + 16 * c4);
          dq[8 * q + c4] =
              good ? make_float4(wj * (__uint_as_float(u[4 * c4]) + l4.x),
                                 wj * (__uint_as_float(u[4 * c4 + 1]) + l4.y),
                                 wj * (__uint_as_float(u[4 * c4 + 2]) + l4.z),
                                 wj * (__uint_as_float(u[4 * c4 + 3]) + l4.w))
                   : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace dsa
