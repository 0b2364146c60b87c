// Backward of the lightning indexer against its KL training target.
//
// The indexer is trained to imitate the main attention's head-summed distribution through a KL
// divergence ("DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek Sparse Attention (DSA)",
// "Training signal"); in the sparse stage both distributions live on the selected keys.  With
// the real-valued inputs q[t,j,:] = s_q[t,j] qh[t,j,:] and k[s,:] = s_k[s] kh[s,:] (the e4m3
// codes times their scales), per query row t over its selected keys e (idx[t,e] >= 0):
//   D[j,e] = q[t,j,:] . k[s_e,:],   S_e = sum_j w[t,j] max(D[j,e], 0)   (the indexer score)
//   pi = softmax(S),   loss_t = sum_e p_e (ln p_e - ln pi_e)            (p = the target row)
//   g_e = dloss_t / dS_e = pi_e sum_f p_f - p_e
//   dw[t,j]    = sum_e g_e max(D[j,e], 0)
//   dq[t,j,:]  = w[t,j] sum_e g_e [D[j,e] > 0] k[s_e,:]
//   dk[s_e,:] += g_e sum_j w[t,j] [D[j,e] > 0] q[t,j,:]   (summed over rows with atomic adds)
// The derivative of max(x, 0) at 0 is taken as 0.
//
// This CUDA-core kernel serves the small indexer shape (4 heads: too narrow an N for an MMA);
// the 64 x 128 shape runs on the tensor cores (indexer_bwd_tc.cuh), which reuses the parameter
// block and the e4m3 decoding below.
//
// Design (CUDA cores, fp32).  One CTA of 256 threads per query row, two CTAs per SM.  The row's
// real-valued queries stay in shared memory (row stride D_I + 1 floats, so that lanes reading
// one dim of consecutive heads hit distinct banks); keys come 64 at a time, decoded from e4m3 and
// scaled into shared memory.  The loops are register-tiled so that shared-memory loads, not
// FMAs, stop being the bound: each 4-dim step of the dot products loads 8 keys (broadcast) and
// 2 heads' queries for 64 FMAs, dk loads the coefficients of 8 keys 4 heads at a time, dq those
// of 8 heads per key.  Pass 1 computes every S_e: warp w takes keys 8w..8w+7 of the chunk, lane
// l heads l and l + 32, and the head sum is a butterfly over the lanes.  Block reductions then
// give max S, the softmax normaliser, sum p, the loss and g.  Pass 2 recomputes D chunk by chunk
// (the same instructions, so the same values and ReLU decisions as pass 1) and forms
// coef[e][j] = g_e w_j [D > 0] in shared memory; dw accumulates in registers, dk (lanes over
// dims, per key) goes out with coalesced atomic adds, and dq (warp = 8 heads, lane = dims
// l + 32 c) accumulates in registers over all chunks.  Chunks without a valid key are skipped.
// Dense mode (no index array): the entries are the row's keys 0..pos(t), at most MAX_K.
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "sm100.cuh"

namespace dsa {

struct IdxBwdParams {
  const uint8_t* q_idx;        // [T, H_I, D_I] e4m3
  const float* q_scale;        // [T, H_I]
  const float* w;              // [T, H_I]
  const uint8_t* k_idx;        // [R, D_I] e4m3
  const float* k_scale;        // [R]
  const int32_t* idx;          // [row_count, topk] logical keys, -1 = unused
  const float* target;         // [row_count, topk]
  const float* sel;            // optional [row_count, topk]: the indexer scores of the selected
                               // keys (the forward's); the softmax is taken over them
  float* loss;                 // [row_count]
  float* dw;                   // [row_count, H_I]
  float* dq;                   // [row_count, H_I, D_I]
  float* dk;                   // [R, D_I], accumulated
  int32_t row_begin, row_count, topk;
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
  int64_t ld_target;           // target row stride (topk; dense: >= every row's key count)
  int32_t dense;               // 1: every prior key of each row (prefill), no idx
};

template <int H_I, int D_I>
struct IdxBwdCfg {
  static constexpr int THREADS = 256;
  static constexpr int CH = 64;                       // keys per chunk
  static constexpr int KPW = CH / 8;                  // keys per warp
  static constexpr int HPL = (H_I + 31) / 32;         // heads per lane (D, coef)
  static constexpr int HPW = (H_I + 7) / 8;           // heads per warp (dq)
  static constexpr int DPL = D_I / 32;                // dims per lane (dq, dk)
  static constexpr int QS = D_I + 1;                  // query row stride in shared memory
  static constexpr int MAX_K = 2048;
  static constexpr int MAX_CH = MAX_K / CH;
  // floats: queries, key chunk, coef (the dw partials reuse it at the end), S / g, w; then
  // ints: physical rows, chunk flags; then 32 floats of reduction scratch.  97 KB at
  // (64, 128): two CTAs per SM.
  static constexpr int SMEM_BYTES =
      4 * (H_I * QS + CH * D_I + CH * H_I + MAX_K + H_I) + 4 * (MAX_K + MAX_CH) + 4 * 32 + 16;
  static_assert(D_I % 32 == 0 && H_I <= 64 && H_I % 4 == 0, "shape");
  static_assert(8 * H_I <= CH * H_I, "dw partials fit the coef buffer");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// 4 e4m3 codes (one 32-bit word, first code in the low byte) -> 4 floats times `scale`
__device__ __forceinline__ float4 decode4_e4m3(uint32_t raw, float scale) {
  const __half2 lo = __half2(__nv_cvt_fp8x2_to_halfraw2(
      static_cast<__nv_fp8x2_storage_t>(raw & 0xFFFFu), __NV_E4M3));
  const __half2 hi = __half2(__nv_cvt_fp8x2_to_halfraw2(
      static_cast<__nv_fp8x2_storage_t>(raw >> 16), __NV_E4M3));
  const float2 a = __half22float2(lo), b = __half22float2(hi);
  return make_float4(a.x * scale, a.y * scale, b.x * scale, b.y * scale);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, m));
  return x;
}

// Block-wide sum or max of one value per thread (256 threads); every thread gets the result.
template <bool kMax>
__device__ __forceinline__ float block_reduce(float x, float* scratch) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  x = kMax ? warp_max(x) : warp_sum(x);
  __syncthreads();   // scratch may still be read by a previous reduction
  if (lane == 0) scratch[warp] = x;
  __syncthreads();
  float y = lane < 8 ? scratch[lane] : (kMax ? -INFINITY : 0.f);
  y = kMax ? warp_max(y) : warp_sum(y);
  return y;
}

template <int H_I, int D_I>
__global__ void __launch_bounds__(256, 2) dsa_indexer_kl_bwd_kernel(const IdxBwdParams p) {
  using C = IdxBwdCfg<H_I, D_I>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* sQ = reinterpret_cast<float*>(smem_raw);     // [H_I][QS]
  float* sK = sQ + H_I * C::QS;                       // [CH][D_I]  (16-byte aligned rows)
  float* sCoef = sK + C::CH * D_I;                    // [CH][H_I]
  float* sG = sCoef + C::CH * H_I;                    // [MAX_K]: S, then g
  float* sDw = sCoef;                                 // [8 warps][H_I], after the last chunk
  float* sW = sG + C::MAX_K;                          // [H_I]
  int32_t* sPhys = reinterpret_cast<int32_t*>(sW + H_I);   // [MAX_K]
  int32_t* sChunk = sPhys + C::MAX_K;                 // [MAX_CH]
  float* sScr = reinterpret_cast<float*>(sChunk + C::MAX_CH);   // [32]

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int r = blockIdx.x;
  const int row = p.row_begin + r;
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
  // entries of the row: the selection (topk slots), or in dense mode its keys 0..pos (at most
  // MAX_K, checked by the caller), padded to whole chunks
  const int K = p.dense ? (min(n_keys, C::MAX_K) + C::CH - 1) / C::CH * C::CH : p.topk;
  const int n_chunks = K / C::CH;

  // ---- queries (real-valued) and weights into shared memory
  {
    const uint8_t* qrow = p.q_idx + static_cast<int64_t>(row) * H_I * D_I;
    for (int u = tid; u < H_I * D_I / 4; u += C::THREADS) {
      const int j = (u * 4) / D_I, i0 = (u * 4) % D_I;
      const float4 f = decode4_e4m3(__ldg(reinterpret_cast<const uint32_t*>(qrow) + u),
                                    __ldg(p.q_scale + static_cast<int64_t>(row) * H_I + j));
      float* dst = sQ + j * C::QS + i0;
      dst[0] = f.x;
      dst[1] = f.y;
      dst[2] = f.z;
      dst[3] = f.w;
    }
    if (tid < H_I) sW[tid] = __ldg(p.w + static_cast<int64_t>(row) * H_I + tid);
  }
  // ---- selected keys -> physical rows (-1: unused or out of range)
  {
    bool bad = false;
    const int32_t* irow = p.dense ? nullptr : p.idx + static_cast<int64_t>(r) * K;
    for (int e = tid; e < K; e += C::THREADS) {
      const int v = p.dense ? (e < n_keys ? e : -1) : __ldg(irow + e);
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
  __syncthreads();
  for (int c = warp; c < n_chunks; c += 8) {
    const bool v = sPhys[c * C::CH + lane] >= 0 || sPhys[c * C::CH + 32 + lane] >= 0;
    const unsigned any = __ballot_sync(0xffffffffu, v);
    if (lane == 0) sChunk[c] = any != 0u;
  }
  __syncthreads();

  // one chunk of keys, decoded and scaled, into sK (unused keys: zeros); consecutive lanes
  // take consecutive 4-code words, so the float4 stores are conflict-free
  auto load_chunk = [&](int c) {
    for (int u = tid; u < C::CH * D_I / 4; u += C::THREADS) {
      const int e = (u * 4) / D_I, i0 = (u * 4) % D_I;
      const int32_t ph = sPhys[c * C::CH + e];
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      if (ph >= 0)
        f = decode4_e4m3(__ldg(reinterpret_cast<const uint32_t*>(
                             p.k_idx + static_cast<int64_t>(ph) * D_I + i0)),
                         __ldg(p.k_scale + ph));
      *reinterpret_cast<float4*>(sK + e * D_I + i0) = f;
    }
  };
  // D[j][e] for this warp's 4 keys and this lane's heads
  auto dots = [&](float (&acc)[C::HPL][C::KPW]) {
#pragma unroll
    for (int hh = 0; hh < C::HPL; ++hh)
#pragma unroll
      for (int kk = 0; kk < C::KPW; ++kk) acc[hh][kk] = 0.f;
#pragma unroll 4
    for (int i = 0; i < D_I; i += 4) {
      float4 kv[C::KPW];
#pragma unroll
      for (int kk = 0; kk < C::KPW; ++kk)
        kv[kk] = *reinterpret_cast<const float4*>(sK + (warp * C::KPW + kk) * D_I + i);
#pragma unroll
      for (int hh = 0; hh < C::HPL; ++hh) {
        const int j = lane + 32 * hh;
        float q0 = 0.f, q1 = 0.f, q2 = 0.f, q3 = 0.f;
        if (j < H_I) {
          const float* qj = sQ + j * C::QS + i;
          q0 = qj[0];
          q1 = qj[1];
          q2 = qj[2];
          q3 = qj[3];
        }
#pragma unroll
        for (int kk = 0; kk < C::KPW; ++kk) {
          float a = acc[hh][kk];
          a = fmaf(q0, kv[kk].x, a);
          a = fmaf(q1, kv[kk].y, a);
          a = fmaf(q2, kv[kk].z, a);
          a = fmaf(q3, kv[kk].w, a);
          acc[hh][kk] = a;
        }
      }
    }
  };

  // ---- pass 1: the scores S_e (given: read them)
  const bool have_sel = p.sel != nullptr && !p.dense;
  if (have_sel)
    for (int e = tid; e < K; e += C::THREADS)
      sG[e] = sPhys[e] >= 0 ? __ldg(p.sel + static_cast<int64_t>(r) * K + e) : -INFINITY;
  for (int c = 0; c < n_chunks && !have_sel; ++c) {
    if (!sChunk[c]) {
      if (tid < C::CH) sG[c * C::CH + tid] = -INFINITY;
      continue;
    }
    load_chunk(c);
    __syncthreads();
    float acc[C::HPL][C::KPW];
    dots(acc);
#pragma unroll
    for (int kk = 0; kk < C::KPW; ++kk) {
      float x = 0.f;
#pragma unroll
      for (int hh = 0; hh < C::HPL; ++hh) {
        const int j = lane + 32 * hh;
        if (j < H_I) x = fmaf(sW[j], fmaxf(acc[hh][kk], 0.f), x);
      }
      x = warp_sum(x);
      const int e = c * C::CH + warp * C::KPW + kk;
      if (lane == 0) sG[e] = sPhys[e] >= 0 ? x : -INFINITY;
    }
    __syncthreads();
  }
  __syncthreads();

  // ---- softmax, loss and g = dloss/dS
  const float* trow = p.target + static_cast<int64_t>(r) * p.ld_target;
  float m = -INFINITY;
  for (int e = tid; e < K; e += C::THREADS) m = fmaxf(m, sG[e]);
  m = block_reduce<true>(m, sScr);
  float z = 0.f, psum = 0.f;
  if (m != -INFINITY)
    for (int e = tid; e < K; e += C::THREADS)
      if (sPhys[e] >= 0) {
        z += expf(sG[e] - m);
        psum += __ldg(trow + e);
      }
  z = block_reduce<false>(z, sScr);
  psum = block_reduce<false>(psum, sScr);
  const float log_z = m == -INFINITY ? 0.f : m + logf(z);
  float l = 0.f;
  for (int e = tid; e < K; e += C::THREADS) {
    float g = 0.f;
    if (sPhys[e] >= 0) {
      const float pe = __ldg(trow + e);
      const float log_pi = sG[e] - log_z;
      if (pe > 0.f) l += pe * (logf(pe) - log_pi);
      g = expf(log_pi) * psum - pe;
    }
    sG[e] = g;
  }
  l = block_reduce<false>(l, sScr);
  if (tid == 0) p.loss[r] = l;
  __syncthreads();

  // ---- pass 2: gradients
  float dwacc[C::HPL];
#pragma unroll
  for (int hh = 0; hh < C::HPL; ++hh) dwacc[hh] = 0.f;
  float dqacc[C::HPW][C::DPL];
#pragma unroll
  for (int h8 = 0; h8 < C::HPW; ++h8)
#pragma unroll
    for (int dd = 0; dd < C::DPL; ++dd) dqacc[h8][dd] = 0.f;

  for (int c = 0; c < n_chunks; ++c) {
    if (!sChunk[c]) continue;
    load_chunk(c);
    __syncthreads();
    float acc[C::HPL][C::KPW];
    dots(acc);
#pragma unroll
    for (int kk = 0; kk < C::KPW; ++kk) {
      const int el = warp * C::KPW + kk;
      const float ge = sG[c * C::CH + el];
#pragma unroll
      for (int hh = 0; hh < C::HPL; ++hh) {
        const int j = lane + 32 * hh;
        if (j < H_I) {
          const float d = acc[hh][kk];
          dwacc[hh] = fmaf(ge, fmaxf(d, 0.f), dwacc[hh]);
          sCoef[el * H_I + j] = d > 0.f ? ge * sW[j] : 0.f;
        }
      }
    }
    __syncwarp();
    // dk of this warp's keys: lanes over dims; coefficients 4 heads at a time
    {
      float kacc[C::KPW][C::DPL];
#pragma unroll
      for (int kk = 0; kk < C::KPW; ++kk)
#pragma unroll
        for (int dd = 0; dd < C::DPL; ++dd) kacc[kk][dd] = 0.f;
      const float* cw = sCoef + warp * C::KPW * H_I;
#pragma unroll 1
      for (int j0 = 0; j0 < H_I; j0 += 4) {
        float4 cf[C::KPW];
#pragma unroll
        for (int kk = 0; kk < C::KPW; ++kk)
          cf[kk] = *reinterpret_cast<const float4*>(cw + kk * H_I + j0);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          float qv[C::DPL];
#pragma unroll
          for (int dd = 0; dd < C::DPL; ++dd) qv[dd] = sQ[(j0 + h) * C::QS + lane + 32 * dd];
#pragma unroll
          for (int kk = 0; kk < C::KPW; ++kk) {
            const float c = h == 0 ? cf[kk].x : h == 1 ? cf[kk].y : h == 2 ? cf[kk].z : cf[kk].w;
#pragma unroll
            for (int dd = 0; dd < C::DPL; ++dd) kacc[kk][dd] = fmaf(c, qv[dd], kacc[kk][dd]);
          }
        }
      }
#pragma unroll
      for (int kk = 0; kk < C::KPW; ++kk) {
        const int32_t ph = sPhys[c * C::CH + warp * C::KPW + kk];
        if (ph < 0) continue;
        float* dst = p.dk + static_cast<int64_t>(ph) * D_I + lane;
#pragma unroll
        for (int dd = 0; dd < C::DPL; ++dd) atomicAdd(dst + 32 * dd, kacc[kk][dd]);
      }
    }
    __syncthreads();   // every warp's coef is in place
    // dq: warp = heads [HPW w, HPW w + HPW), lanes over dims
#pragma unroll 2
    for (int e = 0; e < C::CH; ++e) {
      float kv[C::DPL];
#pragma unroll
      for (int dd = 0; dd < C::DPL; ++dd) kv[dd] = sK[e * D_I + lane + 32 * dd];
      float cf[C::HPW];
      if constexpr (C::HPW % 4 == 0) {   // this warp's heads are whole float4s of the row
#pragma unroll
        for (int q4 = 0; q4 < C::HPW / 4; ++q4) {
          const float4 t =
              *reinterpret_cast<const float4*>(sCoef + e * H_I + warp * C::HPW + 4 * q4);
          cf[4 * q4] = t.x;
          cf[4 * q4 + 1] = t.y;
          cf[4 * q4 + 2] = t.z;
          cf[4 * q4 + 3] = t.w;
        }
      } else {
#pragma unroll
        for (int h8 = 0; h8 < C::HPW; ++h8) {
          const int j = warp * C::HPW + h8;
          cf[h8] = j < H_I ? sCoef[e * H_I + j] : 0.f;
        }
      }
#pragma unroll
      for (int h8 = 0; h8 < C::HPW; ++h8)
#pragma unroll
        for (int dd = 0; dd < C::DPL; ++dd) dqacc[h8][dd] = fmaf(cf[h8], kv[dd], dqacc[h8][dd]);
    }
    __syncthreads();   // sK and sCoef are rewritten by the next chunk
  }

  // ---- outputs
#pragma unroll
  for (int h8 = 0; h8 < C::HPW; ++h8) {
    const int j = warp * C::HPW + h8;
    if (j >= H_I) continue;
    float* dst = p.dq + (static_cast<int64_t>(r) * H_I + j) * D_I + lane;
#pragma unroll
    for (int dd = 0; dd < C::DPL; ++dd) dst[32 * dd] = dqacc[h8][dd];
  }
#pragma unroll
  for (int hh = 0; hh < C::HPL; ++hh) {
    const int j = lane + 32 * hh;
    if (j < H_I) sDw[warp * H_I + j] = dwacc[hh];
  }
  __syncthreads();
  if (tid < H_I) {
    float a = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < 8; ++w8) a += sDw[w8 * H_I + tid];
    p.dw[static_cast<int64_t>(r) * H_I + tid] = a;
  }
}

}  // namespace dsa
