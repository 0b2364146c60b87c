/*
 * CPU oracle for the DSA hot path -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the package's smoke check and the benchmark's CPU-baseline leg may call
 * this code.  It shares nothing with the CUDA path: no headers, helpers or tables.
 *
 * It writes out, plainly and slowly, what the three stages of DeepSeek Sparse Attention
 * compute, in the order the pages give ("FP8 index -> top-k selection -> sparse core
 * attention", "DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek Sparse Attention
 * (DSA)", pipeline summary):
 *
 *   indexer   S[t,s] = s_k[s] * sum_j w[t,j] * s_q[t,j] * ReLU( sum_i qh[t,j,i] * kh[s,i] )
 *             for every prior key s <= pos(t) of the same sequence (the lightning indexer
 *             scores context tokens, same page, "two-stage attention path"; the weighted
 *             sum of ReLU(q.k) over indexer heads is the reading this repository uses)
 *   top-k     the k keys with the largest S; ties go to the smaller key index; when fewer
 *             than k keys precede the query all of them are kept ("top-k=2048", same page,
 *             "Training signal"; "Top-k selector keeps k key-value pairs per query",
 *             maplevalley page, section 1)
 *   attention MLA in MQA mode: every selected latent row is shared by all query heads
 *             (same page, "Instantiation"); logits l_s = sigma * q.kv[s], O = softmax-
 *             weighted sum of the first d_v latent dims, LSE = log sum exp(l_s)
 *
 * The indexer's training signal (same page, "Training signal": the indexer imitates the main
 * attention's head-summed distribution through a KL divergence) is written out too: the target
 * distribution on the selected keys and the loss with its gradients for w, q and k.
 *
 * Floating point: e4m3 and bf16 inputs are decoded exactly; the indexer runs in fp64 (or
 * in fp32 with index-ordered accumulation when asked), attention runs in fp64.  The decode
 * cache append quantises the new token's indexer key per token to e4m3 ("FP8 index", same
 * page, pipeline summary) in fp32, the precision the kernel uses for that decision.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- exact decoding of the input formats ---------------------------------------------- */

/* OCP 8-bit floating point, E4M3 variant: 1 sign bit, 4 exponent bits with bias 7, 3
 * mantissa bits; exponent field 0 encodes subnormals m/8 * 2^-6; S.1111.111 is NaN; there
 * is no infinity, so the largest finite magnitude is 1.75 * 2^8 = 448. */
double dsa_oracle_e4m3_to_f64(uint8_t byte) {
  int sign = byte >> 7;
  int e = (byte >> 3) & 0xF;
  int m = byte & 0x7;
  double v;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0)
    v = ldexp((double)m / 8.0, -6);
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32. */
double dsa_oracle_bf16_to_f64(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double g_e4m3[256];
static void ensure_e4m3_table(void) {
  static int ready = 0;
  if (ready) return;
  for (int b = 0; b < 256; ++b) g_e4m3[b] = dsa_oracle_e4m3_to_f64((uint8_t)b);
  ready = 1;
}

/* ---- indexer ------------------------------------------------------------------------------ */

/* One sequence.  Keys are given in logical order (key s of the sequence at row s of k_fp8);
 * query row r sits at position pos[r] and is scored against keys 0..pos[r].
 *   q_fp8   [n_rows, h_idx, d_idx] e4m3 bytes
 *   q_scale [n_rows, h_idx], w [n_rows, h_idx]
 *   k_fp8   [n_keys, d_idx] e4m3 bytes, k_scale [n_keys]
 *   out     [n_rows, ld_out]; entries s > pos[r] are left untouched
 * fp32_path != 0: the dot products and the head sum are accumulated in binary32 in index
 * order (the arithmetic a single-precision evaluation of the formula performs); otherwise
 * binary64. */
void dsa_oracle_indexer_seq(int n_rows, int h_idx, int d_idx, const uint8_t* q_fp8,
                            const float* q_scale, const float* w, const int32_t* pos,
                            int n_keys, const uint8_t* k_fp8, const float* k_scale,
                            int64_t ld_out, double* out, int fp32_path) {
  ensure_e4m3_table();
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n_rows; ++r) {
    const uint8_t* qr = q_fp8 + (int64_t)r * h_idx * d_idx;
    int last = pos[r] < n_keys - 1 ? pos[r] : n_keys - 1;
    for (int s = 0; s <= last; ++s) {
      const uint8_t* ks = k_fp8 + (int64_t)s * d_idx;
      if (fp32_path) {
        float acc = 0.0f;
        for (int j = 0; j < h_idx; ++j) {
          float dot = 0.0f;
          for (int i = 0; i < d_idx; ++i)
            dot += (float)g_e4m3[qr[j * d_idx + i]] * (float)g_e4m3[ks[i]];
          float relu = dot > 0.0f ? dot : 0.0f;
          acc += w[r * h_idx + j] * q_scale[r * h_idx + j] * relu;
        }
        out[(int64_t)r * ld_out + s] = (double)(k_scale[s] * acc);
      } else {
        double acc = 0.0;
        for (int j = 0; j < h_idx; ++j) {
          double dot = 0.0;
          for (int i = 0; i < d_idx; ++i) dot += g_e4m3[qr[j * d_idx + i]] * g_e4m3[ks[i]];
          double relu = dot > 0.0 ? dot : 0.0;
          acc += (double)w[r * h_idx + j] * (double)q_scale[r * h_idx + j] * relu;
        }
        out[(int64_t)r * ld_out + s] = (double)k_scale[s] * acc;
      }
    }
  }
}

/* ---- top-k -------------------------------------------------------------------------------- */

typedef struct {
  double score;
  int32_t index;
} scored_t;

/* Order: larger score first; equal scores -> smaller index first. */
static int by_score_then_index(const void* a, const void* b) {
  const scored_t* x = (const scored_t*)a;
  const scored_t* y = (const scored_t*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->index > y->index) - (x->index < y->index);
}

/* For each row: keys 0..n_valid[r]-1 of scores[r*ld + s] are candidates.  Writes the
 * min(topk, n_valid) selected key indices in selection order (best first) and pads with
 * -1.  A full sort of the candidates under the order above: plain, not fast. */
void dsa_oracle_topk(int n_rows, int topk, const double* scores, int64_t ld,
                     const int32_t* n_valid, int32_t* idx) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n_rows; ++r) {
    int n = n_valid[r];
    scored_t* c = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
    for (int s = 0; s < n; ++s) {
      c[s].score = scores[(int64_t)r * ld + s];
      c[s].index = s;
    }
    qsort(c, (size_t)n, sizeof(scored_t), by_score_then_index);
    for (int j = 0; j < topk; ++j) idx[(int64_t)r * topk + j] = j < n ? c[j].index : -1;
    free(c);
  }
}

/* ---- sparse MLA attention in MQA mode ------------------------------------------------------ */

/* For each row r and head h, over the physical latent rows rows[r, 0..k) that are >= 0:
 *   l_s = scale * sum_{i<d_qk} q[r,h,i] * kv[s,i]
 *   O[r,h,:] = sum_s exp(l_s - m) kv[s, 0:d_v] / sum_s exp(l_s - m),  m = max_s l_s
 *   LSE[r,h] = m + ln sum_s exp(l_s - m)
 * q and kv are bf16 bit patterns.  A row with no valid entry gets O = 0 and LSE = -inf. */
void dsa_oracle_sparse_mla(int n_rows, int h, int d_qk, int d_v, double scale,
                           const uint16_t* q, const uint16_t* kv, const int64_t* rows, int k,
                           double* out, double* lse) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n_rows; ++r) {
    double* qd = (double*)malloc(sizeof(double) * (size_t)d_qk);
    double* logit = (double*)malloc(sizeof(double) * (size_t)k);
    double* acc = (double*)malloc(sizeof(double) * (size_t)d_v);
    const int64_t* sel = rows + (int64_t)r * k;
    for (int hh = 0; hh < h; ++hh) {
      const uint16_t* qrow = q + ((int64_t)r * h + hh) * d_qk;
      for (int i = 0; i < d_qk; ++i) qd[i] = dsa_oracle_bf16_to_f64(qrow[i]);
      double m = -INFINITY;
      for (int j = 0; j < k; ++j) {
        if (sel[j] < 0) continue;
        const uint16_t* kr = kv + sel[j] * (int64_t)d_qk;
        double dot = 0.0;
        for (int i = 0; i < d_qk; ++i) dot += qd[i] * dsa_oracle_bf16_to_f64(kr[i]);
        logit[j] = scale * dot;
        if (logit[j] > m) m = logit[j];
      }
      double* o = out + ((int64_t)r * h + hh) * d_v;
      if (m == -INFINITY) {
        for (int i = 0; i < d_v; ++i) o[i] = 0.0;
        lse[(int64_t)r * h + hh] = -INFINITY;
        continue;
      }
      double denom = 0.0;
      for (int i = 0; i < d_v; ++i) acc[i] = 0.0;
      for (int j = 0; j < k; ++j) {
        if (sel[j] < 0) continue;
        double p = exp(logit[j] - m);
        const uint16_t* kr = kv + sel[j] * (int64_t)d_qk;
        denom += p;
        for (int i = 0; i < d_v; ++i) acc[i] += p * dsa_oracle_bf16_to_f64(kr[i]);
      }
      for (int i = 0; i < d_v; ++i) o[i] = acc[i] / denom;
      lse[(int64_t)r * h + hh] = m + log(denom);
    }
    free(qd);
    free(logit);
    free(acc);
  }
}

/* ---- indexer training signal --------------------------------------------------------------- */

/* The indexer learns to imitate the main attention's head-summed distribution through a KL
 * divergence ("DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek Sparse Attention (DSA)",
 * "Training signal").  In the sparse stage both distributions live on the selected keys.
 *
 * Target, for each row r over the physical latent rows rows[r, 0..k) that are >= 0:
 *   l_{h,e} = scale * sum_{i<d_qk} q[r,h,i] * kv[rows[r,e], i]
 *   LSE_h   = ln sum_e exp(l_{h,e})                         (over the selection)
 *   t_e     = (1/h) sum_h exp(l_{h,e} - LSE_h)              (each head's distribution sums to 1,
 *                                                            so t does too)
 * Entries with rows < 0 get 0; a row with no valid entry is all 0.  q and kv are bf16 bit
 * patterns; the arithmetic is binary64. */
void dsa_oracle_attn_target(int n_rows, int h, int d_qk, double scale, const uint16_t* q,
                            const uint16_t* kv, const int64_t* rows, int k, double* target) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n_rows; ++r) {
    double* qd = (double*)malloc(sizeof(double) * (size_t)d_qk);
    double* logit = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
    const int64_t* sel = rows + (int64_t)r * k;
    double* t = target + (int64_t)r * k;
    for (int e = 0; e < k; ++e) t[e] = 0.0;
    for (int hh = 0; hh < h; ++hh) {
      const uint16_t* qrow = q + ((int64_t)r * h + hh) * d_qk;
      for (int i = 0; i < d_qk; ++i) qd[i] = dsa_oracle_bf16_to_f64(qrow[i]);
      double m = -INFINITY;
      for (int e = 0; e < k; ++e) {
        if (sel[e] < 0) continue;
        const uint16_t* kr = kv + sel[e] * (int64_t)d_qk;
        double dot = 0.0;
        for (int i = 0; i < d_qk; ++i) dot += qd[i] * dsa_oracle_bf16_to_f64(kr[i]);
        logit[e] = scale * dot;
        if (logit[e] > m) m = logit[e];
      }
      if (m == -INFINITY) continue;
      double z = 0.0;
      for (int e = 0; e < k; ++e)
        if (sel[e] >= 0) z += exp(logit[e] - m);
      const double lse = m + log(z);
      for (int e = 0; e < k; ++e)
        if (sel[e] >= 0) t[e] += exp(logit[e] - lse) / (double)h;
    }
    free(qd);
    free(logit);
  }
}

/* KL loss of the indexer against a target distribution, and its gradients.  Per row r, over
 * the entries e < k with valid[r,e] != 0 (the selected keys), with real-valued inputs (the
 * fp8 codes times their scales):
 *   D_{j,e} = sum_{i<d} q[r,j,i] * keys[r,e,i]
 *   S_e     = sum_j w[r,j] * max(D_{j,e}, 0)                 (the indexer score)
 *   pi      = softmax_e(S)
 *   loss_r  = sum_e p_e (ln p_e - ln pi_e)  with p = target[r, :] and 0 ln 0 = 0
 *   g_e     = dloss/dS_e = pi_e * sum_f p_f - p_e
 *   dw[r,j]      = sum_e g_e max(D_{j,e}, 0)
 *   dq[r,j,:]    = sum_e g_e w[r,j] [D_{j,e} > 0] keys[r,e,:]
 *   dkeys[r,e,:] = sum_j g_e w[r,j] [D_{j,e} > 0] q[r,j,:]
 * (the derivative of max(x, 0) at x = 0 is taken as 0).  Invalid entries get S = -inf and
 * zero gradients.  scores [n_rows, k] receives S.  Binary64 throughout. */
void dsa_oracle_indexer_kl(int n_rows, int h_idx, int d, int k, const double* q,
                           const double* w, const double* keys, const int32_t* valid,
                           const double* target, double* loss, double* scores, double* dw,
                           double* dq, double* dkeys) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n_rows; ++r) {
    const double* qr = q + (int64_t)r * h_idx * d;
    const double* wr = w + (int64_t)r * h_idx;
    const double* kr = keys + (int64_t)r * k * d;
    const int32_t* vr = valid + (int64_t)r * k;
    const double* pr = target + (int64_t)r * k;
    double* sr = scores + (int64_t)r * k;
    double* dot = (double*)malloc(sizeof(double) * (size_t)h_idx * (size_t)(k > 0 ? k : 1));
    double* g = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
    /* scores */
    double m = -INFINITY;
    for (int e = 0; e < k; ++e) {
      sr[e] = -INFINITY;
      if (!vr[e]) continue;
      double acc = 0.0;
      for (int j = 0; j < h_idx; ++j) {
        double dd = 0.0;
        for (int i = 0; i < d; ++i) dd += qr[j * d + i] * kr[(int64_t)e * d + i];
        dot[(int64_t)j * k + e] = dd;
        acc += wr[j] * (dd > 0.0 ? dd : 0.0);
      }
      sr[e] = acc;
      if (acc > m) m = acc;
    }
    /* softmax, loss, dloss/dS */
    double z = 0.0, psum = 0.0, l = 0.0;
    for (int e = 0; e < k; ++e)
      if (vr[e]) {
        z += exp(sr[e] - m);
        psum += pr[e];
      }
    const double logz = (m == -INFINITY) ? 0.0 : m + log(z);
    for (int e = 0; e < k; ++e) {
      g[e] = 0.0;
      if (!vr[e]) continue;
      const double logpi = sr[e] - logz;
      if (pr[e] > 0.0) l += pr[e] * (log(pr[e]) - logpi);
      g[e] = exp(logpi) * psum - pr[e];
    }
    loss[r] = l;
    /* gradients */
    for (int j = 0; j < h_idx; ++j) {
      double a = 0.0;
      for (int e = 0; e < k; ++e)
        if (vr[e]) {
          const double dd = dot[(int64_t)j * k + e];
          a += g[e] * (dd > 0.0 ? dd : 0.0);
        }
      dw[(int64_t)r * h_idx + j] = a;
      for (int i = 0; i < d; ++i) {
        double b = 0.0;
        for (int e = 0; e < k; ++e)
          if (vr[e] && dot[(int64_t)j * k + e] > 0.0) b += g[e] * kr[(int64_t)e * d + i];
        dq[((int64_t)r * h_idx + j) * d + i] = wr[j] * b;
      }
    }
    for (int e = 0; e < k; ++e)
      for (int i = 0; i < d; ++i) {
        double c = 0.0;
        if (vr[e])
          for (int j = 0; j < h_idx; ++j)
            if (dot[(int64_t)j * k + e] > 0.0) c += wr[j] * qr[j * d + i];
        dkeys[((int64_t)r * k + e) * d + i] = g[e] * c;
      }
    free(dot);
    free(g);
  }
}

/* Threads the OpenMP runtime will use (reported beside CPU timings). */
/* ---- per-token e4m3 quantisation (the decode cache append) --------------------------------- */

/* Round-to-nearest-even of a finite |y| <= 448 onto the E4M3 grid, from the format's
 * definition: below 2^-6 the grid is m * 2^-9 (m = 0..8, and m = 8 is the first normal value
 * 2^-6); from 2^e to 2^(e+1) (e = -6..8) it is (1 + m/8) * 2^e, m = 0..7.  Returns the code. */
static uint8_t e4m3_round(float yf) {
  double y = (double)yf;                  /* exact */
  uint8_t sign = 0;
  if (y < 0) { sign = 0x80; y = -y; }
  if (y >= 448.0) return sign | 0x7E;    /* saturate (the caller clamps already) */
  if (y < ldexp(1.0, -6)) {
    double q = y / ldexp(1.0, -9);        /* exact: division by a power of two */
    double f = floor(q);
    double r = q - f;
    double m = (r > 0.5 || (r == 0.5 && fmod(f, 2.0) != 0.0)) ? f + 1.0 : f;
    return sign | (uint8_t)m;             /* m = 8 encodes exponent field 1, mantissa 0 */
  }
  int e;
  frexp(y, &e);                           /* y = fr * 2^e, fr in [0.5, 1) */
  e -= 1;                                 /* y in [2^e, 2^(e+1)) */
  double q = (y / ldexp(1.0, e) - 1.0) * 8.0;   /* exact */
  double f = floor(q);
  double r = q - f;
  int m = (int)f + ((r > 0.5 || (r == 0.5 && ((int)f & 1))) ? 1 : 0);
  if (m == 8) { m = 0; e += 1; }
  return sign | (uint8_t)(((e + 7) << 3) | m);
}

/* Quantise n_rows rows of d fp32 values, each with its own scale: amax = max |x| over the
 * row, scale = amax / 448 in fp32 (1 when amax = 0), y = x / scale in fp32, clamped to
 * [-448, 448], then rounded to the nearest E4M3 value (ties to even).  codes [n_rows, d],
 * scales [n_rows]. */
void dsa_oracle_quantize_e4m3(int n_rows, int d, const float* x, uint8_t* codes, float* scales) {
  for (int r = 0; r < n_rows; ++r) {
    const float* xr = x + (int64_t)r * d;
    float amax = 0.0f;
    for (int i = 0; i < d; ++i) amax = fmaxf(amax, fabsf(xr[i]));
    const float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
    scales[r] = scale;
    for (int i = 0; i < d; ++i) {
      float y = xr[i] / scale;
      if (y > 448.0f) y = 448.0f;
      if (y < -448.0f) y = -448.0f;
      codes[(int64_t)r * d + i] = e4m3_round(y);
    }
  }
}

int dsa_oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
