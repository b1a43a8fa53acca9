/*
 * mla_oracle.c -- plain fp64 CPU oracle for absorbed multi-head latent attention
 * (MLA) decode over a paged latent cache.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load this library. It shares no code, header, table or helper
 * with the CUDA path.
 *
 * What it computes (per batch entry b, query position s, head h):
 *   the absorbed score of "TransMLA: Multi-Head Latent Attention Is All You Need"
 *   (sec. 3.4.5, "The full MLA structure after conversion") and of the TPLA page
 *   (sec. 3.4, "The RoPE handling", the summed content + positional score):
 *
 *     sigma_t = scale * ( q_lat[b,s,h,:] . c_t  +  q_rope[b,s,h,:] . kR_t )
 *     lse     = log sum_t exp(sigma_t)
 *     out     = sum_t exp(sigma_t - lse) * c_t
 *
 *   The cached latent c_t is both the key content and the value (TPLA page,
 *   sec. 3.4, eq. 5: softmax(Q c^T) c W^VO). Tokens are fetched through the block
 *   table: token t of sequence b lives in physical block block_table[b][t / bs],
 *   slot t % bs. With causal set and Sq query tokens, query s sees the first
 *   L - Sq + 1 + s tokens (the Sq new tokens are the last Sq of seq_lens[b]).
 *   Rows that see no token get out = 0 and lse = -inf.
 *
 * The softmax is the two-pass textbook form in fp64 (max, then sum of exponentials),
 * with every stored input decoded exactly to double first (the cache append at the end
 * of this file writes that cache):
 *   f32  -> double (exact), f64 as is,
 *   bf16 -> the fp32 whose upper 16 bits are the pattern (exact),
 *   e4m3 (OCP FP8: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
 *   infinities, S.1111.111 = NaN) -> double from that bit definition, then
 *   multiplied by the token's fp32 scale.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1, OR_E4M3 = 2, OR_F64 = 3 };

enum {
  OR_OK = 0,
  OR_ERR_ARG = 1,
  OR_ERR_BLOCK_ID = 2,
  OR_ERR_SEQ_LEN = 3,
  OR_ERR_NOMEM = 4
};

typedef struct {
  int32_t B, Sq, H, r, d_r;
  int32_t block_size, num_blocks, max_blocks_per_seq;
  int32_t q_dtype;      /* OR_F32 | OR_BF16 | OR_F64 */
  int32_t cache_dtype;  /* OR_F32 | OR_BF16 | OR_F64: [num_blocks, bs, r + d_r];
                           OR_E4M3: codes [num_blocks, bs, r] + bf16 k_rope + f32 scale */
  int32_t causal;
  int32_t reserved;
  double softmax_scale;
  const void* q_lat;          /* [B, Sq, H, r] */
  const void* q_rope;         /* [B, Sq, H, d_r] */
  const void* kv_cache;
  const uint16_t* k_rope_cache; /* e4m3 only: bf16 [num_blocks, bs, d_r] */
  const float* kv_scale;        /* e4m3 only: [num_blocks, bs] */
  const int32_t* block_table;   /* [B, max_blocks_per_seq] */
  const int32_t* seq_lens;      /* [B] */
} mla_oracle_problem;

double mla_oracle_bf16_to_double(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

double mla_oracle_e4m3_to_double(uint8_t code) {
  int sign = code >> 7;
  int e = (code >> 3) & 0xF;
  int m = code & 0x7;
  double v;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);              /* subnormal: m/8 * 2^(1-7) */
  else
    v = ldexp((double)(8 + m), e - 10);    /* (1 + m/8) * 2^(e-7) */
  return sign ? -v : v;
}

static double load_elem(const void* base, int dtype, size_t i) {
  switch (dtype) {
    case OR_F32: return (double)((const float*)base)[i];
    case OR_BF16: return mla_oracle_bf16_to_double(((const uint16_t*)base)[i]);
    case OR_F64: return ((const double*)base)[i];
    default: return NAN;
  }
}

/* Number of tokens query row s of sequence b attends to. */
static int64_t attended(const mla_oracle_problem* p, int64_t L, int s) {
  int64_t n = p->causal ? L - p->Sq + 1 + s : L;
  return n < 0 ? 0 : n;
}

static int check_problem(const mla_oracle_problem* p) {
  if (!p || p->B < 0 || p->Sq < 1 || p->H < 1 || p->r < 1 || p->d_r < 0 || p->block_size < 1 ||
      p->num_blocks < 0 || p->max_blocks_per_seq < 0)
    return OR_ERR_ARG;
  if (p->cache_dtype == OR_E4M3 && (p->d_r > 0 && !p->k_rope_cache)) return OR_ERR_ARG;
  if (p->cache_dtype == OR_E4M3 && !p->kv_scale) return OR_ERR_ARG;
  for (int b = 0; b < p->B; ++b) {
    int64_t L = p->seq_lens[b];
    if (L < 0 || L > (int64_t)p->max_blocks_per_seq * p->block_size) return OR_ERR_SEQ_LEN;
    int64_t nb = (L + p->block_size - 1) / p->block_size;
    for (int64_t i = 0; i < nb; ++i) {
      int32_t blk = p->block_table[(size_t)b * p->max_blocks_per_seq + i];
      if (blk < 0 || blk >= p->num_blocks) return OR_ERR_BLOCK_ID;
    }
  }
  return OR_OK;
}

/* Decode the tokens [t0, t1) of sequence b to double: row k holds c (r) then kR (d_r). */
static void gather_tokens(const mla_oracle_problem* p, int b, int64_t t0, int64_t t1, double* dst) {
  const int D = p->r + p->d_r;
  for (int64_t t = t0; t < t1; ++t) {
    int32_t blk = p->block_table[(size_t)b * p->max_blocks_per_seq + t / p->block_size];
    size_t slot = (size_t)blk * p->block_size + (size_t)(t % p->block_size);
    double* row = dst + (size_t)(t - t0) * D;
    if (p->cache_dtype == OR_E4M3) {
      const uint8_t* codes = (const uint8_t*)p->kv_cache + slot * p->r;
      double sc = (double)p->kv_scale[slot];
      for (int k = 0; k < p->r; ++k) row[k] = mla_oracle_e4m3_to_double(codes[k]) * sc;
      for (int j = 0; j < p->d_r; ++j)
        row[p->r + j] = mla_oracle_bf16_to_double(p->k_rope_cache[slot * p->d_r + j]);
    } else {
      for (int k = 0; k < D; ++k) row[k] = load_elem(p->kv_cache, p->cache_dtype, slot * D + k);
    }
  }
}

/*
 * Query row qrow (= (b * Sq + s) * H + h) against the n decoded tokens in toks (row k:
 * c then kR). sigma is scratch of n. n = 0 gives out = 0, lse = -inf.
 */
static void softmax_row(const mla_oracle_problem* p, size_t qrow, int64_t n, const double* toks, double* sigma,
                        double* out, double* lse) {
  const int D = p->r + p->d_r;
  for (int k = 0; k < p->r; ++k) out[k] = 0.0;
  if (n <= 0) {
    *lse = -INFINITY;
    return;
  }
  double qv_stack[1024];
  double* qv = D <= 1024 ? qv_stack : (double*)malloc(sizeof(double) * D);
  for (int k = 0; k < p->r; ++k) qv[k] = load_elem(p->q_lat, p->q_dtype, qrow * p->r + k);
  for (int j = 0; j < p->d_r; ++j) qv[p->r + j] = load_elem(p->q_rope, p->q_dtype, qrow * p->d_r + j);

  /* pass 1: scores and their maximum */
  double M = -INFINITY;
  for (int64_t t = 0; t < n; ++t) {
    const double* c = toks + (size_t)t * D;
    double content = 0.0, positional = 0.0;
    for (int k = 0; k < p->r; ++k) content += qv[k] * c[k];
    for (int j = 0; j < p->d_r; ++j) positional += qv[p->r + j] * c[p->r + j];
    double sg = p->softmax_scale * (content + positional);
    sigma[t] = sg;
    if (sg > M) M = sg;
  }
  /* pass 2: normaliser, log-sum-exp, weighted sum of latents */
  double Z = 0.0;
  for (int64_t t = 0; t < n; ++t) Z += exp(sigma[t] - M);
  double L = M + log(Z);
  for (int64_t t = 0; t < n; ++t) {
    double w = exp(sigma[t] - L);
    const double* c = toks + (size_t)t * D;
    for (int k = 0; k < p->r; ++k) out[k] += w * c[k];
  }
  *lse = L;
  if (qv != qv_stack) free(qv);
}

/*
 * One (b, s, h) row over the token window [t0, t1) intersected with what the row may
 * attend to. toks holds the decoded tokens [t0, t1). sigma is scratch of t1 - t0.
 */
static void decode_row(const mla_oracle_problem* p, int b, int s, int h, int64_t t0, int64_t t1,
                       const double* toks, double* sigma, double* out, double* lse) {
  int64_t n = attended(p, p->seq_lens[b], s);
  int64_t hi = t1 < n ? t1 : n;
  softmax_row(p, ((size_t)b * p->Sq + s) * p->H + h, hi - t0, toks, sigma, out, lse);
}

/*
 * Full decode, or a window of it: for each b, only tokens [tok_begin[b], tok_end[b])
 * take part (NULL = the whole sequence). Windows give the per-split partial results
 * that a log-sum-exp merge recombines.
 * out: [B, Sq, H, r] double, lse: [B, Sq, H] double.
 */
int mla_oracle_decode_window(const mla_oracle_problem* p, const int64_t* tok_begin,
                             const int64_t* tok_end, double* out, double* lse, int nthreads) {
  int rc = check_problem(p);
  if (rc) return rc;
  const int D = p->r + p->d_r;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  for (int b = 0; b < p->B; ++b) {
    int64_t L = p->seq_lens[b];
    int64_t t0 = tok_begin ? tok_begin[b] : 0;
    int64_t t1 = tok_end ? tok_end[b] : L;
    if (t0 < 0) t0 = 0;
    if (t1 > L) t1 = L;
    if (t1 < t0) t1 = t0;
    double* toks = (double*)malloc(sizeof(double) * (size_t)((t1 - t0) > 0 ? (t1 - t0) : 1) * D);
    if (!toks) return OR_ERR_NOMEM;
    gather_tokens(p, b, t0, t1, toks);
    int nrows = p->Sq * p->H;
    int err = 0;
#pragma omp parallel
    {
      double* sigma = (double*)malloc(sizeof(double) * (size_t)((t1 - t0) > 0 ? (t1 - t0) : 1));
      if (!sigma) {
#pragma omp atomic write
        err = 1;
      } else {
#pragma omp for schedule(dynamic, 1)
        for (int row = 0; row < nrows; ++row) {
          int s = row / p->H, h = row % p->H;
          size_t o = ((size_t)b * p->Sq + s) * p->H + h;
          decode_row(p, b, s, h, t0, t1, toks, sigma, out + o * p->r, lse + o);
        }
        free(sigma);
      }
    }
    free(toks);
    if (err) return OR_ERR_NOMEM;
  }
  return OR_OK;
}

int mla_oracle_decode(const mla_oracle_problem* p, double* out, double* lse, int nthreads) {
  return mla_oracle_decode_window(p, NULL, NULL, out, lse, nthreads);
}

/*
 * Selected rows only: rows[3*i .. 3*i+2] = (b, s, h). out: [n, r], lse: [n].
 * Used to check full-size runs on a sample of output rows.
 */
int mla_oracle_decode_rows(const mla_oracle_problem* p, int n, const int32_t* rows, double* out,
                           double* lse, int nthreads) {
  int rc = check_problem(p);
  if (rc) return rc;
  const int D = p->r + p->d_r;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < n; ++i) {
    int b = rows[3 * i], s = rows[3 * i + 1], h = rows[3 * i + 2];
    if (b < 0 || b >= p->B || s < 0 || s >= p->Sq || h < 0 || h >= p->H) {
#pragma omp atomic write
      err = OR_ERR_ARG;
      continue;
    }
    int64_t L = p->seq_lens[b];
    double* toks = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * D);
    double* sigma = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    if (!toks || !sigma) {
#pragma omp atomic write
      err = OR_ERR_NOMEM;
    } else {
      gather_tokens(p, b, 0, L, toks);
      decode_row(p, b, s, h, 0, L, toks, sigma, out + (size_t)i * p->r, lse + i);
    }
    free(toks);
    free(sigma);
  }
  return err;
}

/*
 * Log-sum-exp merge of n_parts partial results over disjoint token windows:
 *   lse = log sum_i exp(lse_i),  out = sum_i exp(lse_i - lse) * o_i.
 * o_parts: [n_parts, n_rows, r], lse_parts: [n_parts, n_rows].
 */
void mla_oracle_merge(int n_parts, int n_rows, int r, const double* o_parts, const double* lse_parts,
                      double* out, double* lse) {
  for (int row = 0; row < n_rows; ++row) {
    double M = -INFINITY;
    for (int i = 0; i < n_parts; ++i) {
      double v = lse_parts[(size_t)i * n_rows + row];
      if (v > M) M = v;
    }
    for (int k = 0; k < r; ++k) out[(size_t)row * r + k] = 0.0;
    if (M == -INFINITY) {
      lse[row] = -INFINITY;
      continue;
    }
    double Z = 0.0;
    for (int i = 0; i < n_parts; ++i) Z += exp(lse_parts[(size_t)i * n_rows + row] - M);
    double L = M + log(Z);
    for (int i = 0; i < n_parts; ++i) {
      double w = exp(lse_parts[(size_t)i * n_rows + row] - L);
      if (w == 0.0) continue;
      const double* o = o_parts + ((size_t)i * n_rows + row) * r;
      for (int k = 0; k < r; ++k) out[(size_t)row * r + k] += w * o[k];
    }
    lse[row] = L;
  }
}

/* ------------------------------------------------------------------ cache append
 *
 * The producer side of the cache the decode reads ("TransMLA: Multi-Head Latent
 * Attention Is All You Need", sec. 3.4.5: one latent and one decoupled RoPE key per
 * token; the RoPE key is rotated for the token's position, as the "Watching the fusion
 * actually fail, on numbers" passage of the TransMLA & Sparse Latent Attention lesson
 * shows with R(t) on a 2-D toy).
 */

/* fp32 -> OCP e4m3 code, round to nearest with ties to the even code, magnitudes above
 * 448 saturate to 448, NaN -> 0x7F. Plain search over the 127 finite magnitudes. */
uint8_t mla_oracle_e4m3_encode(float x) {
  if (isnan(x)) return 0x7F;
  const uint8_t sign = signbit(x) ? 0x80 : 0x00;
  const double a = fabs((double)x);
  int best = 0;
  double best_err = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    const double err = fabs(mla_oracle_e4m3_to_double((uint8_t)c) - a);
    if (err < best_err || (err == best_err && (c & 1) == 0)) {
      best = c;
      best_err = err;
    }
  }
  return (uint8_t)(sign | best);
}

void mla_oracle_e4m3_encode_n(const float* x, uint8_t* codes, int64_t n) {
  for (int64_t i = 0; i < n; ++i) codes[i] = mla_oracle_e4m3_encode(x[i]);
}

/* fp32 -> bf16 bits, round to nearest even (finite inputs). */
static uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/*
 * For token s of sequence b (pos = seq_lens[b] - Sq + s, block block_table[b][pos / bs],
 * slot pos % bs): store the latent (as given, or as e4m3 codes with the per-token scale
 * max|c| / 448 computed in fp32 and codes e4m3(c / scale) of the fp32 quotient), and the
 * RoPE key, rotated first when rope is set: pairs (x[2i], x[2i+1]) turn by
 * pos * base^(-2i / d_r), in fp64, rounded to fp32 and then to the cache type.
 * Tokens with a bad position or block id are skipped; the first such error is returned.
 */
int mla_oracle_cache_append(int B, int Sq, int r, int d_r, int bs, int num_blocks, int max_blocks,
                            int in_dtype, int cache_dtype, int rope, double rope_base, const void* c_new,
                            const void* k_new, void* cache, uint16_t* k_rope_cache, float* kv_scale,
                            const int32_t* block_table, const int32_t* seq_lens) {
  int err = OR_OK;
  const int D = r + d_r;
  for (int b = 0; b < B; ++b) {
    for (int s = 0; s < Sq; ++s) {
      const int64_t pos = (int64_t)seq_lens[b] - Sq + s;
      if (pos < 0 || pos >= (int64_t)max_blocks * bs) {
        if (!err) err = OR_ERR_SEQ_LEN;
        continue;
      }
      const int32_t blk = block_table[(size_t)b * max_blocks + pos / bs];
      if (blk < 0 || blk >= num_blocks) {
        if (!err) err = OR_ERR_BLOCK_ID;
        continue;
      }
      const size_t slot = (size_t)blk * bs + (size_t)(pos % bs);
      const size_t row = (size_t)b * Sq + s;
      /* latent */
      if (cache_dtype == OR_E4M3) {
        const uint16_t* c = (const uint16_t*)c_new + row * r;
        float amax = 0.f;
        for (int k = 0; k < r; ++k) {
          const float v = (float)mla_oracle_bf16_to_double(c[k]);
          if (fabsf(v) > amax) amax = fabsf(v);
        }
        const float scale = amax / 448.0f;
        uint8_t* codes = (uint8_t*)cache + slot * r;
        for (int k = 0; k < r; ++k) {
          const float v = (float)mla_oracle_bf16_to_double(c[k]);
          codes[k] = mla_oracle_e4m3_encode(scale > 0.f ? v / scale : 0.f);
        }
        kv_scale[slot] = scale;
      } else if (cache_dtype == OR_BF16) {
        memcpy((uint16_t*)cache + slot * D, (const uint16_t*)c_new + row * r, (size_t)r * 2);
      } else {
        memcpy((float*)cache + slot * D, (const float*)c_new + row * r, (size_t)r * 4);
      }
      /* RoPE key */
      for (int j = 0; j < d_r; ++j) {
        double y;
        const double x = load_elem(k_new, in_dtype, row * d_r + j);
        if (rope) {
          const int i = j / 2;
          const double theta = pow(rope_base, -2.0 * i / d_r);
          const double ang = (double)pos * theta;
          const double x0 = load_elem(k_new, in_dtype, row * d_r + 2 * i);
          const double x1 = load_elem(k_new, in_dtype, row * d_r + 2 * i + 1);
          const double cs = cos(ang), sn = sin(ang);
          y = (j % 2 == 0) ? x0 * cs - x1 * sn : x0 * sn + x1 * cs;
        } else {
          y = x;
        }
        const float yf = (float)y;
        if (cache_dtype == OR_F32)
          ((float*)cache)[slot * D + r + j] = yf;
        else if (cache_dtype == OR_BF16)
          ((uint16_t*)cache)[slot * D + r + j] = f32_to_bf16_rne(yf);
        else
          k_rope_cache[slot * d_r + j] = f32_to_bf16_rne(yf);
      }
    }
  }
  return err;
}

/* ------------------------------------------------------------------ per-head products
 *
 * y[m, h, j] = sum_k x[m, h, k] * w[h, k, j] in fp64 from bf16 / f32 / f64 storage: the query
 * absorption (w[h] = W^UK_h) and the output up-projection (w[h] = W^UV_h^T) around the
 * absorbed decode ("TransMLA: Multi-Head Latent Attention Is All You Need", sec. 3.4.5).
 */
void mla_oracle_head_gemm(int rows, int heads, int k, int n, int x_dtype, const void* x, int w_dtype, const void* w,
                          double* y) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int m = 0; m < rows; ++m)
    for (int h = 0; h < heads; ++h) {
      double* yr = y + ((size_t)m * heads + h) * n;
      for (int j = 0; j < n; ++j) yr[j] = 0.0;
      for (int kk = 0; kk < k; ++kk) {
        const double xv = load_elem(x, x_dtype, ((size_t)m * heads + h) * k + kk);
        for (int j = 0; j < n; ++j) yr[j] += xv * load_elem(w, w_dtype, ((size_t)h * k + kk) * n + j);
      }
    }
}

/*
 * ---------------------------------------------------------------------------------
 * DeepSeek Sparse Attention (DSA) over the same paged cache: "TransMLA & Sparse Latent
 * Attention" lesson, Chapter 6 ("The lightning indexer", "Fine-grained token selection")
 * and Chapter 7 ("The indexer keeps its own small cache", "DSA runs in MLA's MQA mode").
 *
 * Indexer score of cached token t for query row (b, s), H^I indexer heads:
 *     I_t = sum_j w[b,s,j] * ReLU( q_j . k_t )
 * q_j = e4m3(q_codes[b,s,j,:]) * q_scale[b,s,j]; k_t = e4m3(k_codes[slot(t),:]) * k_scale[slot(t)].
 * The pages run the indexer in FP8 and give no scale layout; the reading here is one
 * fp32 scale per stored vector (per indexer head of a query, per cached token), the
 * same per-token scheme as the FP8 latent cache. The key side-cache k_codes
 * [num_blocks, bs, d^I] shares the latent cache's block table. Query row s sees the
 * first L - Sq + 1 + s tokens when causal, else all L.
 * scores: [B, Sq, max_seq_len] double; entries past a row's attended count are left
 * as they are.
 */
int mla_oracle_dsa_index(int B, int Sq, int HI, int dI, int bs, int num_blocks, int max_blocks, int causal,
                         int max_seq_len, const uint8_t* q_codes, const float* q_scale, const float* w,
                         const uint8_t* k_codes, const float* k_scale, const int32_t* block_table,
                         const int32_t* seq_lens, double* scores, int nthreads) {
  if (B < 0 || Sq < 1 || HI < 1 || dI < 1 || dI > 1024 || bs < 1 || num_blocks < 0 || max_blocks < 0 ||
      max_seq_len < 0)
    return OR_ERR_ARG;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  for (int b = 0; b < B; ++b) {
    const int64_t L = seq_lens[b];
    if (L < 0 || L > (int64_t)max_blocks * bs || L > max_seq_len) return OR_ERR_SEQ_LEN;
    for (int64_t i = 0; i < (L + bs - 1) / bs; ++i) {
      const int32_t blk = block_table[(size_t)b * max_blocks + i];
      if (blk < 0 || blk >= num_blocks) return OR_ERR_BLOCK_ID;
    }
  }
  double* q = (double*)malloc(sizeof(double) * (size_t)HI * dI);
  if (!q) return OR_ERR_NOMEM;
  for (int b = 0; b < B; ++b) {
    const int64_t L = seq_lens[b];
    for (int s = 0; s < Sq; ++s) {
      int64_t n = causal ? L - Sq + 1 + s : L;
      if (n < 0) n = 0;
      const size_t qrow = (size_t)b * Sq + s;
      for (int j = 0; j < HI; ++j) {
        const double qs = (double)q_scale[qrow * HI + j];
        for (int d = 0; d < dI; ++d)
          q[(size_t)j * dI + d] = mla_oracle_e4m3_to_double(q_codes[(qrow * HI + j) * dI + d]) * qs;
      }
      double* out = scores + qrow * (size_t)max_seq_len;
#pragma omp parallel for schedule(static)
      for (int64_t t = 0; t < n; ++t) {
        const int32_t blk = block_table[(size_t)b * max_blocks + t / bs];
        const size_t slot = (size_t)blk * bs + (size_t)(t % bs);
        const double ks = (double)k_scale[slot];
        double kt[1024];
        for (int d = 0; d < dI; ++d) kt[d] = mla_oracle_e4m3_to_double(k_codes[slot * dI + d]) * ks;
        double I = 0.0;
        for (int j = 0; j < HI; ++j) {
          double dot = 0.0;
          for (int d = 0; d < dI; ++d) dot += q[(size_t)j * dI + d] * kt[d];
          I += (double)w[qrow * HI + j] * (dot > 0.0 ? dot : 0.0);
        }
        out[t] = I;
      }
    }
  }
  free(q);
  return OR_OK;
}

/*
 * MLA decode over selected tokens (Chapter 7, "DSA runs in MLA's MQA mode": the
 * selected cache entries are attended in the absorbed form, one latent shared by every
 * head). Query row (b, s) attends exactly the tokens indices[b, s, 0 .. counts[b, s])
 * of sequence b (positions, mapped through the block table); same score, softmax and
 * value as the dense decode above. indices: [B, Sq, top_k], counts: [B, Sq].
 */
int mla_oracle_decode_sparse(const mla_oracle_problem* p, int top_k, const int32_t* indices,
                             const int32_t* counts, double* out, double* lse, int nthreads) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (top_k < 0) return OR_ERR_ARG;
  const int D = p->r + p->d_r;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  /* the list's tokens, decoded, as a window [0, n) of a one-row-per-token buffer */
  double* toks = (double*)malloc(sizeof(double) * (size_t)(top_k > 0 ? top_k : 1) * D);
  if (!toks) return OR_ERR_NOMEM;
  int err = OR_OK;
  for (int b = 0; b < p->B && !err; ++b) {
    for (int s = 0; s < p->Sq && !err; ++s) {
      const size_t row = (size_t)b * p->Sq + s;
      const int n = counts[row];
      if (n < 0 || n > top_k) {
        err = OR_ERR_ARG;
        break;
      }
      for (int i = 0; i < n; ++i) {
        const int32_t t = indices[row * top_k + i];
        if (t < 0 || t >= p->seq_lens[b]) {
          err = OR_ERR_ARG;
          break;
        }
        gather_tokens(p, b, t, t + 1, toks + (size_t)i * D);
      }
      if (err) break;
#pragma omp parallel
      {
        double* sigma = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        if (!sigma) {
#pragma omp atomic write
          err = OR_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 1)
          for (int h = 0; h < p->H; ++h) {
            const size_t o = row * p->H + h;
            softmax_row(p, o, n, toks, sigma, out + o * p->r, lse + o);
          }
          free(sigma);
        }
      }
    }
  }
  free(toks);
  return err;
}
