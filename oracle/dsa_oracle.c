/*
 * dsa_oracle.c -- plain, slow, fp64 CPU oracle for the DeepSeek Sparse Attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load this library.  It shares no code, header, table or helper with the CUDA path
 * under sparse_attention_06_b200/, and it never includes or links anything from there.
 *
 * What it computes (sources are the web pages on the method, by title and section):
 *   "How GLM5.3 Sparse Attention Affects HBM Memory Usage" (English text of the InferenceX
 *   article "Sparse savings, persistent demand: inside GLM-5.3"), section
 *   "Lightning Indexer": the indexer score of key position s for query t is a weighted sum over
 *   the indexer's query heads of ReLU(q_h . k_s); keys are single-headed; there is no value and
 *   no softmax.  Top-K positions are chosen per query and shared by all attention heads; a query
 *   that sees fewer than K positions keeps all of them (dense).
 *   Same page, section "Sparse MLA" / "MLA Modifications": MLA in MQA mode, P = Q[H, d+r] K^T and
 *   O = P V, where K and V come from the same cached latent row (V is its first d dims).
 *   The softmax itself is the standard scaled-dot-product attention (SDPA) softmax named in the
 *   same article's opening section, "How Sparse Attention Affects DRAM/NAND Memory".
 *
 * Readings taken where the pages are silent (each is also listed in the design notes):
 *   - visibility is causal including the query's own position: query t sees 0..q_pos[t];
 *   - no constant scaling inside the indexer (a caller folds any constant into w);
 *   - e4m3 keys are dequantised as e4m3_value * per-token scale before the dot product, and e4m3
 *     queries as e4m3_value * per-(query, head) scale;
 *   - ties in the top-K are broken by the lower position; -0.0 equals +0.0;
 *   - selected positions are emitted in ascending order, padded with -1 when fewer than K;
 *   - LSE is the natural-log log-sum-exp of the scaled logits.
 *
 * Everything is computed in double from the same quantised inputs the GPU sees.  Loops follow
 * the definitions one-to-one; the only parallelism is OpenMP over independent items: the key
 * positions of a query (indexer), the queries (selection) and the heads of a query (attention).
 * The paged address rule (logical position -> physical row) is the plain one:
 *   row = block_table[req][pos / block_size] * block_size + pos % block_size.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1, OR_E4M3 = 2 };

/* bf16 is the upper half of an IEEE binary32. */
static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* OCP FP8 E4M3 ("fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities;
 * exponent 15 with mantissa 7 is NaN; exponent 0 is subnormal with scale 2^-6. */
double oracle_e4m3_to_double(uint8_t b) {
  int sign = (b >> 7) & 1;
  int e = (b >> 3) & 0xF;
  int m = b & 0x7;
  double v;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0)
    v = ldexp((double)m / 8.0, -6);
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

double oracle_bf16_to_double(uint16_t b) { return bf16_bits_to_double(b); }

static double load_elem(const void* base, int dtype, int64_t i) {
  switch (dtype) {
    case OR_F32: return (double)((const float*)base)[i];
    case OR_BF16: return bf16_bits_to_double(((const uint16_t*)base)[i]);
    case OR_E4M3: return oracle_e4m3_to_double(((const uint8_t*)base)[i]);
  }
  return NAN;
}

static int64_t physical_row(const int32_t* block_table, int max_blocks, int block_size, int req,
                            int64_t pos) {
  int64_t blk = block_table[(int64_t)req * max_blocks + pos / block_size];
  return blk * block_size + pos % block_size;
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * Lightning indexer scores.
 *   out[t, s] = sum_h w[t,h] * max(0, sum_i qhat[t,h,i] * khat[s,i])   for 0 <= s <= q_pos[t]
 *   khat[s,i] = key[row(s), i] * (key dtype is e4m3 ? key_scale[row(s)] : 1)
 *   qhat[t,h,i] = q[t,h,i] * (q dtype is e4m3 ? q_scale[t,h] : 1)
 * Entries s > q_pos[t] are left untouched.
 * q: [T, Hi, Di] of q_dtype; q_scale: [T, Hi] f32 (e4m3 queries only); w: [T, Hi] f32;
 * key pool: [num_blocks * block_size, Di] of k_dtype; key_scale: [num_blocks * block_size] f32
 * (e4m3 only).
 */
void oracle_indexer_scores(int T, const void* q, int q_dtype, const float* q_scale, int Hi, int Di, const float* w,
                           const void* kpool, int k_dtype, const float* key_scale, int block_size,
                           const int32_t* block_table, int max_blocks, const int32_t* q_req,
                           const int32_t* q_pos, double* out, int64_t ld, int nthreads) {
  set_threads(nthreads);
  double* qt = (double*)malloc(sizeof(double) * (size_t)Hi * (size_t)Di);
  for (int t = 0; t < T; ++t) {
    for (int64_t e = 0; e < (int64_t)Hi * Di; ++e) {
      double qs = (q_dtype == OR_E4M3) ? (double)q_scale[(int64_t)t * Hi + e / Di] : 1.0;
      qt[e] = load_elem(q, q_dtype, (int64_t)t * Hi * Di + e) * qs;
    }
    int64_t n = (int64_t)q_pos[t] + 1;
    /* the key positions of one query are independent: they are shared out among the threads */
#pragma omp parallel
    {
      double* khat = (double*)malloc(sizeof(double) * (size_t)Di);
#pragma omp for schedule(static)
      for (int64_t s = 0; s < n; ++s) {
        int64_t row = physical_row(block_table, max_blocks, block_size, q_req[t], s);
        double sc = (k_dtype == OR_E4M3) ? (double)key_scale[row] : 1.0;
        for (int i = 0; i < Di; ++i) khat[i] = load_elem(kpool, k_dtype, row * Di + i) * sc;
        double score = 0.0;
        for (int h = 0; h < Hi; ++h) {
          double dot = 0.0;
          for (int i = 0; i < Di; ++i) dot += qt[(int64_t)h * Di + i] * khat[i];
          double relu = dot > 0.0 ? dot : 0.0;
          score += (double)w[(int64_t)t * Hi + h] * relu;
        }
        out[(int64_t)t * ld + s] = score;
      }
      free(khat);
    }
  }
  free(qt);
}

/* Order used by the selection: higher score first; equal scores -> lower position first. */
typedef struct {
  double score;
  int32_t pos;
} scored_pos;

static int by_score_desc_then_pos(const void* a, const void* b) {
  const scored_pos* x = (const scored_pos*)a;
  const scored_pos* y = (const scored_pos*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->pos > y->pos) - (x->pos < y->pos);
}

static int by_int_asc(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/*
 * Top-K selection.  For query t with n = q_pos[t] + 1 visible positions:
 *   n <= K : all positions 0..n-1 (the dense case);
 *   n >  K : the K positions that come first when 0..n-1 are ordered by (score desc, pos asc).
 * The chosen positions are written ascending into idx[t, 0:K], the rest set to -1.
 */
void oracle_topk(int T, const double* scores, int64_t ld, const int32_t* q_pos, int K,
                 int32_t* idx, int nthreads) {
  set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    int64_t n = (int64_t)q_pos[t] + 1;
    int32_t* out = idx + (int64_t)t * K;
    if (n <= K) {
      for (int64_t j = 0; j < K; ++j) out[j] = j < n ? (int32_t)j : -1;
      continue;
    }
    scored_pos* all = (scored_pos*)malloc(sizeof(scored_pos) * (size_t)n);
    for (int64_t s = 0; s < n; ++s) {
      double v = scores[(int64_t)t * ld + s];
      all[s].score = (v == 0.0) ? 0.0 : v; /* -0.0 and +0.0 are the same score */
      all[s].pos = (int32_t)s;
    }
    qsort(all, (size_t)n, sizeof(scored_pos), by_score_desc_then_pos);
    for (int j = 0; j < K; ++j) out[j] = all[j].pos;
    qsort(out, (size_t)K, sizeof(int32_t), by_int_asc);
    free(all);
  }
}

/*
 * Sparse MLA in MQA mode over the selected latent rows.
 * For query t and head h, over the selected positions j (idx[t, j] >= 0):
 *   logit_j = scale * sum_{i < Dqk} q[t,h,i] * lat[row(idx_j), i]
 *   O[t,h,:] = sum_j softmax(logit)_j * lat[row(idx_j), 0:Dv]
 *   lse[t,h] = log(sum_j exp(logit_j))
 * A query with no selected position gets O = 0 and lse = -inf.
 * q: [T, H, Dqk]; latent pool: [num_blocks * block_size, Dqk]; idx: [T, K].
 */
void oracle_sparse_mla(int T, const void* q, int q_dtype, int H, int Dqk, int Dv,
                       const void* lpool, int l_dtype, int block_size, const int32_t* block_table,
                       int max_blocks, const int32_t* q_req, const int32_t* idx, int K,
                       double scale, double* out, double* lse, int nthreads) {
  set_threads(nthreads);
  int64_t* rows = (int64_t*)malloc(sizeof(int64_t) * (size_t)K);
  double* lat = (double*)malloc(sizeof(double) * (size_t)K * (size_t)Dqk);
  for (int t = 0; t < T; ++t) {
    int nsel = 0;
    for (int j = 0; j < K; ++j) {
      int32_t p = idx[(int64_t)t * K + j];
      if (p >= 0) rows[nsel++] = physical_row(block_table, max_blocks, block_size, q_req[t], p);
    }
    for (int j = 0; j < nsel; ++j)
      for (int i = 0; i < Dqk; ++i) lat[(int64_t)j * Dqk + i] = load_elem(lpool, l_dtype, rows[j] * Dqk + i);
    /* the heads of one query are independent: they are shared out among the threads */
#pragma omp parallel
    {
      double* logit = (double*)malloc(sizeof(double) * (size_t)(nsel > 0 ? nsel : 1));
      double* qh = (double*)malloc(sizeof(double) * (size_t)Dqk);
#pragma omp for schedule(static)
      for (int h = 0; h < H; ++h) {
        double* o = out + ((int64_t)t * H + h) * Dv;
        for (int i = 0; i < Dqk; ++i) qh[i] = load_elem(q, q_dtype, ((int64_t)t * H + h) * Dqk + i);
        if (nsel == 0) {
          for (int c = 0; c < Dv; ++c) o[c] = 0.0;
          if (lse) lse[(int64_t)t * H + h] = -INFINITY;
          continue;
        }
        double m = -INFINITY;
        for (int j = 0; j < nsel; ++j) {
          double dot = 0.0;
          for (int i = 0; i < Dqk; ++i) dot += qh[i] * lat[(int64_t)j * Dqk + i];
          logit[j] = scale * dot;
          if (logit[j] > m) m = logit[j];
        }
        double z = 0.0;
        for (int c = 0; c < Dv; ++c) o[c] = 0.0;
        for (int j = 0; j < nsel; ++j) {
          double p = exp(logit[j] - m);
          z += p;
          for (int c = 0; c < Dv; ++c) o[c] += p * lat[(int64_t)j * Dqk + c];
        }
        for (int c = 0; c < Dv; ++c) o[c] /= z;
        if (lse) lse[(int64_t)t * H + h] = m + log(z);
      }
      free(qh);
      free(logit);
    }
  }
  free(lat);
  free(rows);
}
