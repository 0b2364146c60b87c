// Backward of the lightning indexer against its KL training target, on the tensor cores
// (indexer shape 64 heads x 128 dims).  It computes what the CUDA-core kernel in indexer_bwd.cuh
// computes ("DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek Sparse Attention (DSA)",
// "Training signal"; the formulas are stated there), with the three contractions of each row
// as tcgen05 MMAs over 128-key tiles of its selection:
//   D^T  = Kh Qh^T        e4m3, M = 128 keys, N = 64 heads, K = 128 dims (the indexer's shape)
//   dk   = A1 Qh          bf16, M = 128 keys, N = 128 dims, K = 64 heads;
//                         A1[e][j] = g_e w_j s_q,j [D > 0], from Tensor Memory
//   dq^T += Kh^T B2       bf16, M = 128 dims, N = 64 heads, K = 128 keys, accumulated over the
//                         row's tiles; B2[e][j] = g_e s_k,e [D > 0]; Kh^T from Tensor Memory
// Qh and Kh (e4m3 codes) are exact in bf16; the scales and g travel in the coefficients, each
// split into a bf16 pair hi + lo (hi = bf16(x), lo = bf16(x - hi)), so a coefficient keeps 16
// significant bits and the gradients stay at fp32-accumulation accuracy even where g cancels.
//
// One CTA per query row (1 per SM: it allocates all 512 TMEM columns).  Warp 0 issues the MMAs,
// warp 1 owns TMEM, warps 2-3 gather the selected key rows (16-byte cp.async into 128-byte-
// swizzled tiles, two stages; unused keys are zero-filled), warps 4-7 are the epilogue with
// thread = TMEM lane.  Pass 1 runs D^T for every tile and the epilogue forms the scores S
// (thread = key), keeping per thread the running softmax statistics of its keys (max, the sum
// of exp(S - max), and the target's sum, sum p S and sum p ln p); the 128 epilogue threads then
// combine them into the normaliser and the loss.  No per-key value is stored, so a row may have
// any number of entries.  Pass 2 runs D^T again per tile, recomputes S with the same
// instructions (so the same value and ReLU decisions), forms g; the epilogue writes A1 (TMEM,
// thread = key), B2 (shared memory, row = key) and Kh^T (TMEM, thread = dim, read column-wise
// out of the key tile), sums dw over the tile's keys with a butterfly across lanes, and after
// the dk/dq MMAs adds its key's dk row to global memory with 16-byte atomic adds.  At the end
// thread = dim writes dq.  Every wait is bounded.
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
  static constexpr int STAGES = 2;
  static constexpr int THREADS = 256;
  static constexpr int TILE_BYTES = BK * D;        // e4m3 key rows, 16 KB
  // Tensor Memory columns
  static constexpr int D_COL = 0;                  // D^T [128 keys x 64 heads] fp32
  static constexpr int DK_COL = 64;                // dk tile [128 keys x 128 dims] fp32
  static constexpr int DQ_COL = 192;               // dq^T [128 dims x 64 heads] fp32 (whole row)
  static constexpr int A1_COL = 256;               // A1 hi [+0, 32) and lo [+32, 64): bf16 pairs
  static constexpr int KT_COL = 320;               // Kh^T [128 dims x 128 keys]: bf16 pairs
  static constexpr int TMEM_COLS = 512;
  // shared memory, from a 1024-byte-aligned base
  static constexpr int OFF_Q8 = 0;                             // [64 heads][128 B] e4m3 K-major
  static constexpr int OFF_QB = OFF_Q8 + H * D;                // [2 dim blocks][64 heads][128 B]
  static constexpr int OFF_KT = OFF_QB + 2 * H * 128;          // [STAGES][128 keys][128 B] e4m3
  static constexpr int OFF_B2 = OFF_KT + STAGES * TILE_BYTES;  // [hi, lo][128 keys][128 B] bf16
  static constexpr int OFF_PHYS = OFF_B2 + 2 * BK * 128;       // [MAX_K] i32 (selected keys)
  static constexpr int OFF_TILES = OFF_PHYS + 4 * MAX_K;       // [MAX_TILES] i32
  static constexpr int OFF_W = OFF_TILES + 4 * MAX_TILES;      // [64] w
  static constexpr int OFF_SQ = OFF_W + 4 * H;                 // [64] s_q
  static constexpr int OFF_DWP = OFF_SQ + 4 * H;               // [4 warps][64] dw partials
  static constexpr int OFF_SCR = OFF_DWP + 4 * 4 * H;          // [32] reduction scratch
  static constexpr int OFF_BAR = OFF_SCR + 4 * 32;             // barriers
  static constexpr int N_BAR = 16;
  static constexpr int USED = OFF_BAR + 8 * N_BAR;
  // at least 116 KB, so that one CTA runs per SM (its TMEM allocation never waits)
  static constexpr int SMEM_BYTES = 1024 + (USED > 116 * 1024 ? USED : 116 * 1024);
  static_assert(OFF_QB % 1024 == 0 && OFF_KT % 1024 == 0 && OFF_B2 % 1024 == 0, "tiles");
  static_assert(OFF_BAR % 8 == 0, "barriers");
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

__global__ void __launch_bounds__(256, 1) dsa_indexer_kl_bwd_tc_kernel(const IdxBwdParams p) {
  using C = KlTcCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ8 = smem + C::OFF_Q8;
  uint8_t* sQb = smem + C::OFF_QB;
  uint8_t* sKt = smem + C::OFF_KT;
  uint8_t* sB2 = smem + C::OFF_B2;
  int32_t* sPhys = reinterpret_cast<int32_t*>(smem + C::OFF_PHYS);
  int32_t* sTiles = reinterpret_cast<int32_t*>(smem + C::OFF_TILES);
  float* sW = reinterpret_cast<float*>(smem + C::OFF_W);
  float* sSq = reinterpret_cast<float*>(smem + C::OFF_SQ);
  float* sDwp = reinterpret_cast<float*>(smem + C::OFF_DWP);
  float* sScr = reinterpret_cast<float*>(smem + C::OFF_SCR);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;            // [2] 64 gathering threads (each when its copies land)
  uint64_t* kempty = bars + 2;      // [2] 128 epilogue threads: the key tile is no longer read
  uint64_t* d_full = bars + 4;      // D^T MMA commit
  uint64_t* d_empty = bars + 5;     // 128 epilogue threads: D^T read
  uint64_t* coef_full = bars + 6;   // 128 epilogue threads: A1, B2, Kh^T written
  uint64_t* mma_done = bars + 7;    // dk / dq MMA commit
  uint64_t* dk_empty = bars + 8;    // 128 epilogue threads: dk tile read
  uint64_t* ep_bar = bars + 9;      // 128 epilogue threads meet
  uint64_t* fin = bars + 10;        // the MMA issuer's last commit
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

  // ---- prologue: queries (e4m3 K-major for D^T; bf16 MN-major for dk), w, s_q, key rows
  const uint8_t* qrow = p.q_idx + static_cast<int64_t>(row) * C::H * C::D;
  for (int u = tid; u < C::H * 8; u += C::THREADS) {
    const int j = u >> 3, c = u & 7;
    *reinterpret_cast<uint4*>(sQ8 + sw128_offset(j, c)) =
        __ldg(reinterpret_cast<const uint4*>(qrow + j * C::D + c * 16));
  }
  for (int u = tid; u < C::H * 16; u += C::THREADS) {
    const int j = u >> 4, dc = u & 15;             // head j, dims [8 dc, 8 dc + 8)
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(qrow + j * C::D + dc * 8));
    const float4 f0 = decode4_e4m3(raw.x, 1.f), f1 = decode4_e4m3(raw.y, 1.f);
    *reinterpret_cast<uint4*>(sQb + (dc >> 3) * (C::H * 128) + sw128_offset(j, dc & 7)) =
        make_uint4(pack_bf16(f0.x, f0.y), pack_bf16(f0.z, f0.w), pack_bf16(f1.x, f1.y),
                   pack_bf16(f1.z, f1.w));
  }
  if (tid < C::H) {
    sW[tid] = __ldg(p.w + static_cast<int64_t>(row) * C::H + tid);
    sSq[tid] = __ldg(p.q_scale + static_cast<int64_t>(row) * C::H + tid);
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&full[i]), 64);
      mbar_init(smem_u32(&kempty[i]), 128);
    }
    mbar_init(smem_u32(d_full), 1);
    mbar_init(smem_u32(d_empty), 128);
    mbar_init(smem_u32(coef_full), 128);
    mbar_init(smem_u32(mma_done), 1);
    mbar_init(smem_u32(dk_empty), 128);
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

  if (warp == 0) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_d = idesc_f32acc(0 /* e4m3 */, 128, 64, 0, 0);
      constexpr uint32_t id_dk = idesc_f32acc(1 /* bf16 */, 128, 128, 0, 1);
      constexpr uint32_t id_dq = idesc_f32acc(1 /* bf16 */, 128, 64, 0, 1);
      const uint32_t q8 = smem_u32(sQ8), qb = smem_u32(sQb), b2 = smem_u32(sB2);
      bool ok = true;
      for (int it = 0; it < steps && ok; ++it) {
        const int s = it % C::STAGES;
        ok = mbar_wait(smem_u32(&full[s]), (it / C::STAGES) & 1, &abort_s);
        if (ok && it >= 1) ok = mbar_wait(smem_u32(d_empty), (it - 1) & 1, &abort_s);
        if (!ok) break;
        tc_fence_after();
        fence_proxy_async_smem();   // the key tile was written by cp.async
        const uint32_t kt = smem_u32(sKt + s * C::TILE_BYTES);
#pragma unroll
        for (int k = 0; k < C::D / 32; ++k)
          umma_e4m3(tmem + C::D_COL, sdesc_sw128(kt + k * 32, 16, 1024),
                    sdesc_sw128(q8 + k * 32, 16, 1024), id_d, k > 0);
        umma_commit(smem_u32(d_full));
        if (it < n) continue;
        // pass 2: dk = A1 Qh and dq^T += Kh^T B2 for this tile
        const int i2 = it - n;
        ok = mbar_wait(smem_u32(coef_full), i2 & 1, &abort_s);
        if (ok && i2 >= 1) ok = mbar_wait(smem_u32(dk_empty), (i2 - 1) & 1, &abort_s);
        if (!ok) break;
        tc_fence_after();
        fence_proxy_async_smem();   // B2 was written with st.shared
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int k = 0; k < C::H / 16; ++k)
            umma_bf16_ts(tmem + C::DK_COL, tmem + C::A1_COL + 32 * h + 8 * k,
                         sdesc_sw128(qb + k * 16 * 128, C::H * 128, 1024), id_dk, (h | k) != 0);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int k = 0; k < C::BK / 16; ++k)
            umma_bf16_ts(tmem + C::DQ_COL, tmem + C::KT_COL + 8 * k,
                         sdesc_sw128(b2 + h * C::BK * 128 + k * 16 * 128, C::BK * 128, 1024),
                         id_dq, (i2 | h | k) != 0);
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
    // ------------------------------------------------------------ key gather
    // thread pt copies 16-byte chunk (pt & 7) of rows (pt >> 3) + 8 q of every tile
    const int pt = tid - 64;
    const int c = pt & 7, r0 = pt >> 3;
    bool ok = true;
    for (int it = 0; it < steps && ok; ++it) {
      const int s = it % C::STAGES;
      if (it >= C::STAGES &&
          !warp_mbar_wait(smem_u32(&kempty[s]), ((it / C::STAGES) - 1) & 1, &abort_s)) {
        ok = false;
        break;
      }
      const int tile = tile_at(it % n);
      const uint32_t dst = smem_u32(sKt + s * C::TILE_BYTES);
#pragma unroll 4
      for (int q = 0; q < C::BK / 8; ++q) {
        const int rr = r0 + 8 * q;
        const int64_t ph = phys_at(tile * C::BK + rr);
        const void* src = ph >= 0 ? static_cast<const void*>(p.k_idx + static_cast<int64_t>(ph) *
                                                                         C::D + c * 16)
                                  : static_cast<const void*>(p.k_idx);
        cp_async_16(dst + sw128_offset(rr, c), src, ph >= 0 ? 16u : 0u);   // unused: zeros
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
    const float* trow = p.target + static_cast<int64_t>(r) * p.ld_target;
    // (explicitly rounded products: pass 2 must get the bits of pass 1, so the compiler may not
    // fuse them into the arithmetic that follows either call)
    auto score = [&](const uint32_t (&du)[2][32], int64_t ph) -> float {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < C::H; ++j)
        acc = fmaf(__fmul_rn(sW[j], sSq[j]), fmaxf(__uint_as_float(du[j >> 5][j & 31]), 0.f),
                   acc);
      return __fmul_rn(__ldg(p.k_scale + ph), acc);
    };
    float m = -INFINITY, z = 0.f, psum = 0.f, sps = 0.f, splp = 0.f;
    for (int it = 0; it < n && ok; ++it) {
      const int s = it % C::STAGES;
      ok = warp_mbar_wait(smem_u32(d_full), it & 1, &abort_s);
      if (!ok) break;
      tc_fence_after();
      uint32_t du[2][32];
      tmem_ld32(la + C::D_COL, du[0]);
      tmem_ld32(la + C::D_COL + 32, du[1]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(d_empty));
      mbar_arrive(smem_u32(&kempty[s]));
      const int e = tile_at(it) * C::BK + et;
      const int64_t ph = phys_at(e);
      if (ph >= 0) {
        const float S = score(du, ph);
        if (S > m) {
          z = z * expf(m - S) + 1.f;
          m = S;
        } else {
          z += expf(S - m);
        }
        const float pe = __ldg(trow + e);
        psum += pe;
        sps += pe * S;
        if (pe > 0.f) splp += pe * logf(pe);
      }
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

    // ---- pass 2: coefficients, dw, dk; dq accumulates in TMEM
    const int h0 = warp_sum64_first(lane);   // this lane's two heads of the warp's dw sums
    float dw0 = 0.f, dw1 = 0.f;
    for (int i2 = 0; i2 < n && ok; ++i2) {
      const int it = n + i2, s = it % C::STAGES;
      ok = warp_mbar_wait(smem_u32(d_full), it & 1, &abort_s);
      if (!ok) break;
      tc_fence_after();
      uint32_t du[2][32];
      tmem_ld32(la + C::D_COL, du[0]);
      tmem_ld32(la + C::D_COL + 32, du[1]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(d_empty));
      const int e = tile_at(i2) * C::BK + et;
      const int64_t ph = phys_at(e);
      // g = pi psum - p, from the same score as in pass 1 (0 for unused entries)
      const float g = ph >= 0 ? expf(score(du, ph) - log_z) * psum - __ldg(trow + e) : 0.f;
      const float gsk = ph >= 0 ? g * __ldg(p.k_scale + ph) : 0.f;
      // dw: g s_k max(D, 0) summed over the tile's keys (s_q applied at the end)
      {
        float v[64];
#pragma unroll
        for (int j = 0; j < C::H; ++j) v[j] = gsk * fmaxf(__uint_as_float(du[j >> 5][j & 31]), 0.f);
        warp_sum64(v, lane);
        dw0 += v[0];
        dw1 += v[1];
      }
      // A1 = g w_j s_q,j [D > 0] (hi, lo) into TMEM, this key's lane
      {
        uint32_t ahi[32], alo[32];
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) {
          const int j = 2 * c2;
          const float x0 = __uint_as_float(du[j >> 5][j & 31]) > 0.f ? g * sW[j] * sSq[j] : 0.f;
          const float x1 =
              __uint_as_float(du[(j + 1) >> 5][(j + 1) & 31]) > 0.f ? g * sW[j + 1] * sSq[j + 1]
                                                                     : 0.f;
          split_bf16(x0, x1, ahi[c2], alo[c2]);
        }
        tmem_st32(la + C::A1_COL, ahi);
        tmem_st32(la + C::A1_COL + 32, alo);
      }
      // B2 = g s_k [D > 0] (hi, lo): row et of the two B2 tiles
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int j = 8 * c8 + 2 * q;
          const float y0 = __uint_as_float(du[j >> 5][j & 31]) > 0.f ? gsk : 0.f;
          const float y1 = __uint_as_float(du[(j + 1) >> 5][(j + 1) & 31]) > 0.f ? gsk : 0.f;
          split_bf16(y0, y1, hw[q], lw[q]);
        }
        *reinterpret_cast<uint4*>(sB2 + sw128_offset(et, c8)) =
            make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(sB2 + C::BK * 128 + sw128_offset(et, c8)) =
            make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      // Kh^T into TMEM: this thread is dim et; column c holds keys 2c, 2c + 1 (exact in bf16).
      // The tile's own barrier (already complete) orders the cp.async data before these reads.
      ok = warp_mbar_wait(smem_u32(&full[s]), (it / C::STAGES) & 1, &abort_s);
      if (!ok) break;
      {
        const uint8_t* tb = sKt + s * C::TILE_BYTES;
        const uint32_t chunk = static_cast<uint32_t>(et) >> 4, byte = et & 15;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t kw[32];
#pragma unroll
          for (int c2 = 0; c2 < 32; ++c2) {
            const int k0 = 64 * hh + 2 * c2;
            const uint32_t b0 = tb[sw128_offset(k0, chunk) + byte];
            const uint32_t b1 = tb[sw128_offset(k0 + 1, chunk) + byte];
            const __half2 hv = __half2(__nv_cvt_fp8x2_to_halfraw2(
                static_cast<__nv_fp8x2_storage_t>(b0 | (b1 << 8)), __NV_E4M3));
            const float2 f = __half22float2(hv);
            kw[c2] = pack_bf16(f.x, f.y);
          }
          tmem_st32(la + C::KT_COL + 32 * hh, kw);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();   // B2 is read by the tensor cores
      tc_fence_before();
      mbar_arrive(smem_u32(&kempty[s]));
      mbar_arrive(smem_u32(coef_full));
      // dk row of this key, added to global memory
      ok = warp_mbar_wait(smem_u32(mma_done), i2 & 1, &abort_s);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < C::D / 32; ++q) {
        uint32_t u[32];
        tmem_ld32(la + C::DK_COL + 32 * q, u);
        tmem_wait_ld();
        if (ph >= 0) {
          float4* dst = reinterpret_cast<float4*>(p.dk + static_cast<int64_t>(ph) * C::D + 32 * q);
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4)
            atomicAdd(dst + c4, make_float4(__uint_as_float(u[4 * c4]), __uint_as_float(u[4 * c4 + 1]),
                                            __uint_as_float(u[4 * c4 + 2]),
                                            __uint_as_float(u[4 * c4 + 3])));
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(dk_empty));
    }
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
    // ---- dq[j][d] = w_j dq^T[d][j]: this thread is dim et
    float* dq = p.dq + static_cast<int64_t>(r) * C::H * C::D + et;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      uint32_t u[32];
      tmem_ld32(la + C::DQ_COL + 32 * hh, u);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int jj = 32 * hh + j;
        dq[jj * C::D] = (ok && n > 0) ? sW[jj] * __uint_as_float(u[j]) : 0.f;
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
