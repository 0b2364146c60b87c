// Lightning indexer (stage 1): FP8 e4m3 scores of query rows against their prior keys.
//
//   S[t,s] = k_scale[s] * sum_j c[t,j] * ReLU( q[t,j,:] . k[s,:] ),  c[t,j] = w[t,j] * q_scale[t,j]
//
// ("FP8 index -> top-k selection -> sparse core attention", "DeepSeek V3.2-Exp Cuts Long-Context
// Costs with DeepSeek Sparse Attention (DSA)", pipeline summary; "Lightning Indexer", maplevalley
// page, section 1.)
//
// One CTA (grid x = query group, y = key split) takes one query group (QPG rows of the same
// sequence) and a contiguous range of 128-key tiles.  The contraction is swapped so that keys are the MMA's M dimension:
//   D[key, (row, head)] = K_tile[128 x D_I] * Q_group[N x D_I]^T,   N = QPG * H_I
// with e4m3 operands in 128-byte (or 32-byte for D_I = 32) swizzled shared memory and an fp32
// accumulator in Tensor Memory (TMEM lane = key).  Each epilogue thread then owns one key and
// reduces its row's heads with no cross-thread traffic: per head a max (the ReLU) and half of a
// packed fp32x2 FMA (two heads per instruction).
//
// Roles: warp 0 issues TMA (Q once, then per tile two 64-row key boxes plus a bulk copy of each
// box's k_scale), warp 1 issues the tcgen05.mma, warp 2 owns the TMEM allocation, warp 3
// computes c[t,j] (and in decode then issues the tiles of odd index while warp 0 issues the
// even ones: the key stream's rate grows with the threads that issue copies), warps 4.. run the
// epilogue.  Key stages are a ring of STAGES buffers; the
// accumulators are a ring of ACC buffers in TMEM so the epilogue of tile i overlaps the MMA of
// later tiles.  Decode (one query row, N = 64) runs two epilogue warpgroups on alternate tiles;
// prefill (N = 256) splits each tile's columns over four warpgroups, one query row each.
//
// Fused first digit of the top-k (when `hist` is given): as it writes a score, each epilogue
// thread also counts it in its query row's histogram of the top 11 bits of the order-preserving
// key (the first radix digit the top-k selects on), kept in shared memory; at the end the CTA
// adds the non-zero bins into the row's global histogram.  The top-k then starts from exact
// per-row counts and classifies the slab in a single pass.
#pragma once
#include "sm100.cuh"

namespace dsa {

struct IndexerParams {
  const float* q_scale;   // [T, H_I]
  const float* w;         // [T, H_I]
  const float* k_scale;   // [num_kv_rows], or null: paged decode with each block's 64 scales
                          // stored right after its 64 key rows (k_blocks)
  const uint8_t* k_blocks;  // interleaved layout: [num_kv_rows / 64][64 * D_I + 64 * 4] bytes
  float* scores;          // row `out_row0` of the output slab
  int64_t ld;
  int32_t* status;
  int32_t decode;         // 1: one query row per sequence (decode), 0: prefill segment
  // prefill segment: rows [row0, row0 + nrows) of one sequence; row0 sits at position pos0;
  // key s of the sequence is packed row key0 + s.
  // decode: rows [row0, row0 + nrows) are sequences row0.. (one row each)
  int32_t row0, nrows, pos0, key0;
  int32_t out_row0;       // slab row of `row0`
  const int32_t* seq_lens;
  const int32_t* block_table;
  int32_t max_blocks;
  int32_t kv_stride;      // decode without block table: sequence b starts at row b * kv_stride
  int32_t max_seqlen;     // decode: a seq_lens entry above this is clamped and reported
  int64_t num_kv_rows;
  int32_t tiles_per_split;
  uint32_t* hist;         // optional: [slab rows][kIdxHistBins] first-digit counts (added to)
};

constexpr int kIdxHistBins = 2048;   // top 11 bits of the order-preserving score key

// Order-preserving 32-bit key of a score (unsigned order = float order, -0 folded onto +0).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0) u = 0;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int H_I, int D_I, int QPG>
struct IndexerCfg {
  static constexpr int N = H_I * QPG;                 // MMA N: (row, head) columns
  static constexpr int STAGES = QPG == 1 ? 5 : 8;
  // decode streams its keys from two producer warps (tiles of even and odd index), which keeps
  // more page copies moving than one issuing thread does
  static constexpr int PRODUCERS = QPG == 1 ? 2 : 1;
  static constexpr int ACC = QPG == 1 ? 4 : 2;        // TMEM accumulator ring
  static constexpr int EPI_WARPS = QPG == 1 ? 8 : 16;    // prefill: one query row per warpgroup
  static constexpr bool TILE_SPLIT = QPG == 1;        // warpgroups take alternate tiles
  static constexpr int EPI_PER_TILE = TILE_SPLIT ? 4 : EPI_WARPS;   // warps reading one tile
  static constexpr int THREADS = (4 + EPI_WARPS) * 32;
  static constexpr int TILE_BYTES = 128 * D_I;        // 128 keys
  static constexpr int Q_BYTES = N * D_I;
  static constexpr int KSTEPS = D_I / 32;             // one e4m3 MMA consumes K = 32
  static constexpr uint32_t LAYOUT = D_I == 128 ? kSwizzle128B : kSwizzle32B;
  static constexpr uint32_t SBO = 8 * D_I;            // next 8-row group
  static constexpr int TMEM_COLS = ACC * N;
  static constexpr int SCALE_FLOATS = 2 * 80;         // per stage: 2 boxes x (64 + slack)
  // per query row of the group, the first-digit histogram (full shapes; the 64-row groups of
  // the small shape have no room for it and run the top-k's own histogram instead)
  static constexpr bool HIST = QPG <= 4;
  static constexpr int HIST_BYTES = HIST ? QPG * kIdxHistBins * 4 : 0;
  static constexpr int SMEM_BYTES =
      1024 + Q_BYTES + STAGES * TILE_BYTES + STAGES * SCALE_FLOATS * 4 + STAGES * 2 * 16 +
      N * 4 + 512 + HIST_BYTES;
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "MMA N");
  static_assert(TMEM_COLS == 128 || TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM columns");
  static_assert(Q_BYTES % 1024 == 0 && TILE_BYTES % 1024 == 0, "1024-byte aligned tiles");
};

template <int H_I, int D_I, int QPG>
__global__ void __launch_bounds__(IndexerCfg<H_I, D_I, QPG>::THREADS, QPG == 1 ? 2 : 1)
    dsa_indexer_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap qmap, const IndexerParams p) {
  using C = IndexerCfg<H_I, D_I, QPG>;
  constexpr int N = C::N;
  wait_prior_grid();   // (launched early: anything before it in the stream is complete here)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::Q_BYTES;
  float* sScale = reinterpret_cast<float*>(sK + C::STAGES * C::TILE_BYTES);  // [STAGES][2][80]
  // per stage and 64-key half: the cache row of the half's first key, where its scale sits in
  // the stage's scale buffer, and how many of the half's scales were copied there
  int64_t* sRow0 = reinterpret_cast<int64_t*>(sScale + C::STAGES * C::SCALE_FLOATS);  // [STAGES][2]
  int32_t* sFirst = reinterpret_cast<int32_t*>(sRow0 + C::STAGES * 2);   // [STAGES][2]
  int32_t* sValid = sFirst + C::STAGES * 2;                               // [STAGES][2]
  float* sC = reinterpret_cast<float*>(sValid + C::STAGES * 2);
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(sC + N) + 7) & ~uintptr_t(7));
  uint64_t* full = bars;                      // [STAGES] key tile (and its scales) landed
  uint64_t* empty = bars + C::STAGES;         // [STAGES] tile consumed: MMA + epilogue (scales)
  uint64_t* tfull = empty + C::STAGES;        // [ACC] accumulator ready
  uint64_t* tempty = tfull + C::ACC;          // [ACC] accumulator drained by the epilogue
  uint64_t* qbar = tempty + C::ACC;           // Q group landed
  uint64_t* done = qbar + 1;                  // every MMA of this CTA completed
  uint32_t* sHist = reinterpret_cast<uint32_t*>(done + 1);   // [QPG][kIdxHistBins]
  const bool hist_on = C::HIST && p.hist != nullptr;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int last_s[2];   // the last tile each producer issued (-1: none)

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---- geometry of this CTA's group (uniform across the CTA)
  int n_keys, grow0, rows_in_group, pos_first;
  int64_t seq_base = 0;   // decode contiguous: first physical row of the sequence
  int b = 0;
  if (p.decode) {
    b = p.row0 + blockIdx.x;
    n_keys = p.seq_lens[b];
    if (n_keys > p.max_seqlen) {
      if (threadIdx.x == 0 && p.status) atomicOr(p.status, kStatusBadIndex);
      n_keys = p.max_seqlen;
    }
    grow0 = b;
    rows_in_group = 1;
    pos_first = n_keys - 1;
    seq_base = static_cast<int64_t>(b) * p.kv_stride;
    if (n_keys <= 0) return;
  } else {
    grow0 = p.row0 + blockIdx.x * QPG;
    rows_in_group = min(QPG, p.row0 + p.nrows - grow0);
    pos_first = p.pos0 + (grow0 - p.row0);
    n_keys = pos_first + rows_in_group;       // keys 0 .. last row's position
  }
  const int n_tiles_all = (n_keys + 127) / 128;
  const int t_begin = blockIdx.y * p.tiles_per_split;
  const int t_end = min(t_begin + p.tiles_per_split, n_tiles_all);
  if (t_begin >= t_end) return;
  const int n_tiles = t_end - t_begin;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1 + C::EPI_PER_TILE);
    }
    for (int i = 0; i < C::ACC; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), C::TILE_SPLIT ? 4 : C::EPI_WARPS);
    }
    mbar_init(smem_u32(qbar), 1);
    mbar_init(smem_u32(done), 1);
    abort_s = 0;
    fence_mbar_init();
  }
  if (hist_on)
    for (int i = threadIdx.x; i < C::HIST_BYTES / 4; i += C::THREADS) sHist[i] = 0;
  if (warp == 2) tmem_alloc(smem_u32(&tmem_base_s), C::TMEM_COLS);
  if (warp == 3) {
    for (int i = lane; i < N; i += 32) {
      int r = i / H_I, j = i % H_I;
      float c = 0.f;
      if (r < rows_in_group) {
        int64_t row = grow0 + r;
        c = p.w[row * H_I + j] * p.q_scale[row * H_I + j];
      }
      sC[i] = c;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;

  if (warp == 0 || (C::PRODUCERS > 1 && warp == 3)) {
    // ------------------------------------------------------------------ TMA producers
    // producer pr issues tiles pr, pr + PRODUCERS, ... (warp 3 has finished c[t,j] above)
    const int pr = warp == 0 ? 0 : 1;
    int last = -1;
    if (lane == 0) {
      // decode streams the key cache once: evict-first, so that the score slab the top-k reads
      // next stays in L2
      const uint64_t pol = l2_evict_first();
      tma_prefetch_desc(&kmap);
      if (pr == 0) {
        tma_prefetch_desc(&qmap);
        mbar_arrive_expect_tx(smem_u32(qbar), C::Q_BYTES);
        tma_load_2d(smem_u32(sQ), &qmap, smem_u32(qbar), 0, grow0 * H_I);
      }
      const int n_blocks = (n_keys + 63) / 64;
      for (int it = pr; it < n_tiles; it += C::PRODUCERS) {
        const int s = it % C::STAGES;
        if (it >= C::STAGES &&
            !mbar_wait(smem_u32(&empty[s]), ((it / C::STAGES) - 1) & 1, &abort_s)) {
          abort_s = 1;
          if (p.status) atomicOr(p.status, kStatusTimeout);
          break;
        }
        const int tile = t_begin + it;
        float* sbuf = sScale + s * C::SCALE_FLOATS;
        uint32_t bytes;
        if (!p.decode) {
          // prefill: the tile's 128 keys are contiguous rows; one box and one scale copy
          const int64_t y = static_cast<int64_t>(p.key0) + tile * 128;
          const int64_t a0 = y & ~int64_t(3);
          const int64_t avail = p.num_kv_rows - a0;
          const uint32_t sb = static_cast<uint32_t>((avail < 132 ? avail : int64_t(132)) / 4 * 16);
          const int lead = static_cast<int>(y - a0);
          for (int hlf = 0; hlf < 2; ++hlf) {
            sRow0[s * 2 + hlf] = y + hlf * 64;
            sFirst[s * 2 + hlf] = lead + hlf * 64;
            sValid[s * 2 + hlf] = static_cast<int32_t>(sb / 4) - lead - hlf * 64;
          }
          bytes = 128 * D_I + sb;
          mbar_arrive_expect_tx(smem_u32(&full[s]), bytes);
          tma_load_2d(smem_u32(sK + s * C::TILE_BYTES), &kmap, smem_u32(&full[s]), 0,
                      static_cast<int32_t>(y));
          if (sb > 0) bulk_load_g2s(smem_u32(sbuf), p.k_scale + a0, sb, smem_u32(&full[s]));
        } else {
          int64_t y[2];
          bool ok[2];
          for (int hlf = 0; hlf < 2; ++hlf) {
            const int blk = tile * 2 + hlf;
            ok[hlf] = blk < n_blocks;
            if (p.block_table != nullptr) {
              int64_t id = ok[hlf] ? p.block_table[static_cast<int64_t>(b) * p.max_blocks + blk] : 0;
              if (ok[hlf] && (id < 0 || (id + 1) * 64 > p.num_kv_rows)) {
                if (p.status) atomicOr(p.status, kStatusBadIndex);
                ok[hlf] = false;
              }
              y[hlf] = ok[hlf] ? id * 64 : 0;
            } else {
              y[hlf] = seq_base + blk * 64;
            }
          }
          if (p.k_scale == nullptr) {
            // interleaved blocks: 64 key rows (one 3-D box) and their 64 scales, contiguous
            constexpr int64_t kBlockBytes = 64 * (D_I + 4);
            bytes = 0;
            for (int hlf = 0; hlf < 2; ++hlf) {
              sRow0[s * 2 + hlf] = y[hlf];
              sFirst[s * 2 + hlf] = hlf * 80;
              sValid[s * 2 + hlf] = ok[hlf] ? 64 : 0;
              bytes += ok[hlf] ? 64 * D_I + 256 : 0;
            }
            mbar_arrive_expect_tx(smem_u32(&full[s]), bytes);
            for (int hlf = 0; hlf < 2; ++hlf) {
              if (!ok[hlf]) continue;
              const int64_t blk = y[hlf] / 64;
              tma_load_3d_hint(smem_u32(sK + s * C::TILE_BYTES + hlf * 64 * D_I), &kmap,
                               smem_u32(&full[s]), 0, 0, static_cast<int32_t>(blk), pol);
              bulk_load_g2s_hint(smem_u32(sbuf + hlf * 80),
                                 p.k_blocks + blk * kBlockBytes + 64 * D_I, 256,
                                 smem_u32(&full[s]), pol);
            }
          } else {
          // each box's 64 scales: a 16-byte-aligned superset of the rows, inside the cache
          uint32_t sb[2];
          int64_t a0[2];
          for (int hlf = 0; hlf < 2; ++hlf) {
            a0[hlf] = y[hlf] & ~int64_t(3);
            const int64_t avail = p.num_kv_rows - a0[hlf];
            sb[hlf] = ok[hlf] ? static_cast<uint32_t>((avail < 68 ? avail : int64_t(68)) / 4 * 16) : 0u;
            const int lead = static_cast<int>(y[hlf] - a0[hlf]);
            sRow0[s * 2 + hlf] = y[hlf];
            sFirst[s * 2 + hlf] = hlf * 80 + lead;
            sValid[s * 2 + hlf] = static_cast<int32_t>(sb[hlf] / 4) - lead;
          }
          bytes = (ok[0] ? 64 * D_I : 0) + (ok[1] ? 64 * D_I : 0) + sb[0] + sb[1];
          mbar_arrive_expect_tx(smem_u32(&full[s]), bytes);
          for (int hlf = 0; hlf < 2; ++hlf) {
            if (ok[hlf])
              tma_load_2d_hint(smem_u32(sK + s * C::TILE_BYTES + hlf * 64 * D_I), &kmap,
                               smem_u32(&full[s]), 0, static_cast<int32_t>(y[hlf]), pol);
            if (sb[hlf] > 0)
              bulk_load_g2s_hint(smem_u32(sbuf + hlf * 80), p.k_scale + a0[hlf], sb[hlf],
                                 smem_u32(&full[s]), pol);
          }
          }
        }
        last = it;
      }
    }
    // drain: never leave a copy in flight into shared memory of an exiting CTA.  Each stage
    // waits for the last tile issued into it (every earlier use was consumed before that tile
    // could be issued, so only this phase can be outstanding).
    if constexpr (C::PRODUCERS == 1) {
      if (lane == 0)
        for (int it = max(0, last + 1 - C::STAGES); it <= last; ++it)
          mbar_wait(smem_u32(&full[it % C::STAGES]), (it / C::STAGES) & 1, nullptr);
    } else {
      if (lane == 0) last_s[pr] = last;
      __syncwarp();
      named_bar_sync(1, 64);                   // both producer warps are done issuing
      if (pr == 0 && lane == 0)
        for (int st = 0; st < C::STAGES; ++st) {
          int t_last = -1;
          for (int q = 0; q < C::PRODUCERS; ++q)
            for (int t = last_s[q]; t >= 0 && t > last_s[q] - C::PRODUCERS * C::STAGES;
                 t -= C::PRODUCERS)
              if (t % C::STAGES == st) {
                t_last = max(t_last, t);
                break;
              }
          if (t_last >= 0)
            mbar_wait(smem_u32(&full[st]), (t_last / C::STAGES) & 1, nullptr);
        }
    }
    if (pr == 0 && lane == 0) mbar_wait(smem_u32(qbar), 0, nullptr);
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f32acc(0 /* e4m3 */, 128, N, 0, 0);
      bool ok = mbar_wait(smem_u32(qbar), 0, &abort_s);
      for (int it = 0; ok && it < n_tiles; ++it) {
        const int s = it % C::STAGES;
        const int a = it % C::ACC;
        ok = mbar_wait(smem_u32(&full[s]), (it / C::STAGES) & 1, &abort_s);
        if (ok && it >= C::ACC)
          ok = mbar_wait(smem_u32(&tempty[a]), ((it / C::ACC) - 1) & 1, &abort_s);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kaddr = smem_u32(sK + s * C::TILE_BYTES);
        const uint32_t qaddr = smem_u32(sQ);
#pragma unroll
        for (int k = 0; k < C::KSTEPS; ++k)
          umma_e4m3(tmem + a * N, sdesc(kaddr + k * 32, 16, C::SBO, C::LAYOUT),
                    sdesc(qaddr + k * 32, 16, C::SBO, C::LAYOUT), idesc, k > 0);
        umma_commit(smem_u32(&empty[s]));
        umma_commit(smem_u32(&tfull[a]));
      }
      if (!ok) {
        abort_s = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
      }
      umma_commit(smem_u32(done));
      mbar_wait(smem_u32(done), 0, nullptr);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    constexpr int PARTS = C::TILE_SPLIT ? 1 : C::EPI_WARPS / 4;
    constexpr int COLS = N / PARTS;          // columns this warp reduces
    const int quad = warp & 3;               // TMEM lanes 32*quad .. 32*quad+31
    const int grp = (warp - 4) / 4;          // warpgroup
    const int part = C::TILE_SPLIT ? 0 : grp;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint64_t slab_pol = l2_evict_last();   // the decode slab stays in L2 for the top-k
    for (int it = C::TILE_SPLIT ? grp : 0; it < n_tiles; it += C::TILE_SPLIT ? 2 : 1) {
      const int a = it % C::ACC;
      const int s = it % C::STAGES;
      if (!mbar_wait(smem_u32(&tfull[a]), (it / C::ACC) & 1, &abort_s)) {
        abort_s = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      // the tile's scales came with its keys: observe that phase of full[s] (the stage is not
      // refilled before this warp releases it below)
      if (!mbar_wait(smem_u32(&full[s]), (it / C::STAGES) & 1, &abort_s)) {
        abort_s = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
        break;
      }
      const int kin = quad * 32 + lane;        // key within the tile
      const int key = (t_begin + it) * 128 + kin;
      const int hb = kin >> 6;
      const int j = kin & 63;
      float ks = 0.f;
      if (key < n_keys) {
        if (j < sValid[s * 2 + hb]) {
          ks = sScale[s * C::SCALE_FLOATS + sFirst[s * 2 + hb] + j];
        } else {                               // the last rows of the cache: not bulk-copied
          const int64_t row = sRow0[s * 2 + hb] + j;
          ks = p.k_scale != nullptr && row >= 0 && row < p.num_kv_rows ? __ldg(p.k_scale + row)
                                                                          : 0.f;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
      if constexpr (!C::TILE_SPLIT && H_I >= 32 && H_I % 32 == 0) {
        // all of this warp's columns in one TMEM round trip; the accumulator is free again
        // before the arithmetic starts
        constexpr int NCH = COLS / 32;
        uint32_t r[NCH][32];
#pragma unroll
        for (int c = 0; c < NCH; ++c) tmem_ld32(lane_addr + a * N + part * COLS + c * 32, r[c]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&tempty[a]));
        constexpr int CPR = H_I / 32;          // chunks per query row
#pragma unroll
        for (int q = 0; q < NCH / CPR; ++q) {
          // heads in pairs: one packed fp32x2 FMA per two heads (ReLU stays scalar)
          float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
          for (int c = q * CPR; c < (q + 1) * CPR; ++c) {
            const float4* cc = reinterpret_cast<const float4*>(sC + part * COLS + c * 32);
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const float4 c4 = cc[j / 4];
              a01 = __ffma2_rn(make_float2(c4.x, c4.y),
                               make_float2(fmaxf(__uint_as_float(r[c][j + 0]), 0.f),
                                           fmaxf(__uint_as_float(r[c][j + 1]), 0.f)),
                               a01);
              a23 = __ffma2_rn(make_float2(c4.z, c4.w),
                               make_float2(fmaxf(__uint_as_float(r[c][j + 2]), 0.f),
                                           fmaxf(__uint_as_float(r[c][j + 3]), 0.f)),
                               a23);
            }
          }
          const int rr = (part * COLS) / H_I + q;
          if (rr < rows_in_group && key <= pos_first + rr) {
            const float sc = ks * ((a01.x + a01.y) + (a23.x + a23.y));
            p.scores[static_cast<int64_t>(p.out_row0 + (grow0 - p.row0) + rr) * p.ld + key] = sc;
            if (hist_on) atomicAdd(&sHist[rr * kIdxHistBins + (order_key(sc) >> 21)], 1u);
          }
        }
        continue;
      }
      float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);   // heads in pairs
#pragma unroll 1
      for (int c0 = 0; c0 < COLS; c0 += 32) {
        const int col = part * COLS + c0;
        uint32_t r[32];
        tmem_ld32(lane_addr + a * N + col, r);
        tmem_wait_ld();
        const float4* cc = reinterpret_cast<const float4*>(sC + col);
        if constexpr (H_I >= 32) {
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 c4 = cc[j / 4];
            a01 = __ffma2_rn(make_float2(c4.x, c4.y),
                             make_float2(fmaxf(__uint_as_float(r[j + 0]), 0.f),
                                         fmaxf(__uint_as_float(r[j + 1]), 0.f)),
                             a01);
            a23 = __ffma2_rn(make_float2(c4.z, c4.w),
                             make_float2(fmaxf(__uint_as_float(r[j + 2]), 0.f),
                                         fmaxf(__uint_as_float(r[j + 3]), 0.f)),
                             a23);
          }
          if ((col + 32) % H_I == 0) {       // a query row's heads are complete
            const int rr = col / H_I;
            const float acc = (a01.x + a01.y) + (a23.x + a23.y);
            a01 = make_float2(0.f, 0.f);
            a23 = make_float2(0.f, 0.f);
            if (rr < rows_in_group && key <= pos_first + rr) {
              const float sc = ks * acc;
              float* dst = p.scores + static_cast<int64_t>(p.out_row0 + (grow0 - p.row0) + rr) * p.ld + key;
              if (C::TILE_SPLIT) st_global_hint(dst, sc, slab_pol);   // decode: read next
              else *dst = sc;
              if (hist_on) atomicAdd(&sHist[rr * kIdxHistBins + (order_key(sc) >> 21)], 1u);
            }
          }
        } else {
#pragma unroll
          for (int q = 0; q < 32 / H_I; ++q) {
            float sacc = 0.f;
#pragma unroll
            for (int j = 0; j < H_I; ++j)
              sacc = fmaf(sC[col + q * H_I + j], fmaxf(__uint_as_float(r[q * H_I + j]), 0.f), sacc);
            const int rr = col / H_I + q;
            if (rr < rows_in_group && key <= pos_first + rr)
              p.scores[static_cast<int64_t>(p.out_row0 + (grow0 - p.row0) + rr) * p.ld + key] =
                  ks * sacc;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[a]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (hist_on) {
    // this CTA's counts into the rows' global histograms (only the bins it saw)
    for (int i = threadIdx.x; i < rows_in_group * kIdxHistBins; i += C::THREADS) {
      const uint32_t v = sHist[i];
      if (v != 0) {
        const int rr = i / kIdxHistBins;
        atomicAdd(p.hist + static_cast<int64_t>(p.out_row0 + (grow0 - p.row0) + rr) * kIdxHistBins +
                      (i % kIdxHistBins),
                  v);
      }
    }
  }
}

}  // namespace dsa
