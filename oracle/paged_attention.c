/*
 * Paged decode attention, fp64 CPU reference ("the oracle").
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no source
 * with the CUDA path and includes none of its headers.
 *
 * What it computes (FlashInfer README, "core features" 1-3 and the
 * single-request decode usage example; flashinfer-cubin registry page,
 * quickstart names kv_indptr / kv_indices / last_page_len / kv_layout):
 * for every request b and query head hq, with kv head h = hq / (Hq / Hkv)
 * (grouped-query heads in contiguous groups):
 *
 *   n_b   = kv_indptr[b+1] - kv_indptr[b]                 pages of request b
 *   L_b   = 0 if n_b == 0 else (n_b - 1) * P + last_page_len[b]
 *   row_t = kv_indices[kv_indptr[b] + t / P] * P + t % P  pool row of token t
 *   K_t   = k_pool[row_t, h, :],  V_t = v_pool[row_t, h, :]   (NHD pool)
 *   s_t   = sm_scale * sum_d q[b, hq, d] * K_t[d]
 *   lse   = M + ln(sum_t exp(s_t - M)),   M = max_t s_t     (natural log)
 *   o[d]  = sum_t exp(s_t - lse) * V_t[d]
 *
 * An empty request (L_b = 0) gives o = 0 and lse = -inf.  The fp16 / bf16
 * inputs are widened to fp64 exactly; all arithmetic is fp64 in plain
 * token order.  Work is spread over POSIX threads by (b, hq) row only.
 *
 * Low-precision KV cache (README core feature 3: efficient kernels for
 * low-precision attention for compressed KV-Cache): the pools may hold
 * 8-bit floats (OCP FP8 E4M3 without infinities, or E5M2) with one scale
 * for K and one for V; the cached value is scale * code, and q stays fp16 /
 * bf16.
 *
 * Rotary positions on the fly (README usage example: decode with LLaMA-style
 * RoPE, pos_encoding_mode="ROPE_LLAMA"), when rope_theta > 0: before the dot
 * product q is rotated to its position L_b - 1 (the new token is the last in
 * the cache) and key t to position t; element pairs (d, d + D/2) turn by
 * pos * rope_theta^(-2d/D).  Values are not rotated.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int f = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(f + 1024), e - 25); /* (1 + f/1024) * 2^(e-15) */
  return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32. */
static double bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float x;
  memcpy(&x, &u, sizeof x);
  return (double)x;
}

static double widen(uint16_t x, int dtype) { return dtype ? bf16_to_f64(x) : f16_to_f64(x); }

/* OCP FP8 E4M3 ("FN" variant): 1 sign bit, 4 exponent bits (bias 7), 3
 * fraction bits; no infinities, exponent and fraction all ones is NaN, so
 * the largest value is 448. */
static double e4m3_to_f64(uint8_t c) {
  int sign = (c >> 7) & 1;
  int e = (c >> 3) & 0xf;
  int f = c & 0x7;
  double v;
  if (e == 0xf && f == 0x7)
    v = NAN;
  else if (e == 0)
    v = ldexp((double)f, -9); /* subnormal: f/8 * 2^-6 */
  else
    v = ldexp((double)(f + 8), e - 10); /* (1 + f/8) * 2^(e-7) */
  return sign ? -v : v;
}

/* OCP FP8 E5M2: 1 sign bit, 5 exponent bits (bias 15), 2 fraction bits, with
 * IEEE infinities and NaNs. */
static double e5m2_to_f64(uint8_t c) {
  int sign = (c >> 7) & 1;
  int e = (c >> 2) & 0x1f;
  int f = c & 0x3;
  double v;
  if (e == 0)
    v = ldexp((double)f, -16); /* subnormal: f/4 * 2^-14 */
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(f + 4), e - 17); /* (1 + f/4) * 2^(e-15) */
  return sign ? -v : v;
}

/* kv_fmt: -1 = the 16-bit q dtype, 0 = E4M3, 1 = E5M2. */
static double widen8(uint8_t c, int kv_fmt) { return kv_fmt ? e5m2_to_f64(c) : e4m3_to_f64(c); }

/* Exposed so that the tests can pin the 8-bit widening against torch. */
double oracle_widen8(uint8_t x, int32_t kv_fmt) { return widen8(x, kv_fmt); }

/* Exposed so that the tests can pin the widening against numpy / torch. */
double oracle_widen(uint16_t x, int32_t dtype) { return widen(x, dtype); }

typedef struct {
  const uint16_t *q;
  const void *k_pool, *v_pool;
  const int32_t *kv_indptr, *kv_indices, *last_page_len;
  int32_t batch, num_qo_heads, num_kv_heads, head_dim, page_size, dtype, kv_fmt;
  double sm_scale, k_scale, v_scale, rope_theta;
  const int64_t *rows;
  int64_t n_rows;
  double *out_o, *out_lse;
  int64_t next; /* next row to claim, guarded by lock */
  pthread_mutex_t lock;
  int error;
} job_t;

/* Element i of a K or V pool, widened (and scaled, for 8-bit pools). */
static double kv_elem(const job_t *J, const void *pool, int64_t i, double scale) {
  if (J->kv_fmt < 0) return widen(((const uint16_t *)pool)[i], J->dtype);
  return scale * widen8(((const uint8_t *)pool)[i], J->kv_fmt);
}

/* Rotate x (D elements) to position pos: pairs (d, d + D/2) by pos * theta^(-2d/D). */
static void rope(double *x, int D, double pos, double theta) {
  const int half = D / 2;
  for (int d = 0; d < half; ++d) {
    const double a = pos * pow(theta, -2.0 * d / D);
    const double c = cos(a), sn = sin(a);
    const double x0 = x[d], x1 = x[d + half];
    x[d] = x0 * c - x1 * sn;
    x[d + half] = x1 * c + x0 * sn;
  }
}

static void one_row(job_t *J, int64_t r, int64_t out_index, double *s, double *q) {
  const int32_t Hq = J->num_qo_heads, Hkv = J->num_kv_heads, D = J->head_dim, P = J->page_size;
  const int64_t b = r / Hq, hq = r % Hq, h = hq / (Hq / Hkv);
  double *o = J->out_o + out_index * D;
  const int64_t n_b = (int64_t)J->kv_indptr[b + 1] - J->kv_indptr[b];
  const int64_t L = n_b > 0 ? (n_b - 1) * P + J->last_page_len[b] : 0;

  for (int d = 0; d < D; ++d) o[d] = 0.0;
  if (L == 0) {
    J->out_lse[out_index] = -INFINITY;
    return;
  }
  for (int d = 0; d < D; ++d) q[d] = widen(J->q[(b * Hq + hq) * D + d], J->dtype);
  const int rotary = J->rope_theta > 0.0;
  if (rotary) rope(q, D, (double)(L - 1), J->rope_theta);
  double *kr = q + D; /* room for one rotated key */

  /* scores */
  double M = -INFINITY;
  for (int64_t t = 0; t < L; ++t) {
    int64_t row = (int64_t)J->kv_indices[J->kv_indptr[b] + t / P] * P + t % P;
    const int64_t k0 = (row * Hkv + h) * D;
    double acc = 0.0;
    if (rotary) {
      for (int d = 0; d < D; ++d) kr[d] = kv_elem(J, J->k_pool, k0 + d, J->k_scale);
      rope(kr, D, (double)t, J->rope_theta);
      for (int d = 0; d < D; ++d) acc += q[d] * kr[d];
    } else {
      for (int d = 0; d < D; ++d) acc += q[d] * kv_elem(J, J->k_pool, k0 + d, J->k_scale);
    }
    s[t] = J->sm_scale * acc;
    if (s[t] > M) M = s[t];
  }
  /* log-sum-exp */
  double S = 0.0;
  for (int64_t t = 0; t < L; ++t) S += exp(s[t] - M);
  double lse = M + log(S);
  J->out_lse[out_index] = lse;
  /* softmax-weighted values */
  for (int64_t t = 0; t < L; ++t) {
    int64_t row = (int64_t)J->kv_indices[J->kv_indptr[b] + t / P] * P + t % P;
    const int64_t v0 = (row * Hkv + h) * D;
    double w = exp(s[t] - lse);
    for (int d = 0; d < D; ++d) o[d] += w * kv_elem(J, J->v_pool, v0 + d, J->v_scale);
  }
}

static int64_t max_len(const job_t *J) {
  int64_t m = 0;
  for (int32_t b = 0; b < J->batch; ++b) {
    int64_t n = (int64_t)J->kv_indptr[b + 1] - J->kv_indptr[b];
    int64_t L = n > 0 ? (n - 1) * J->page_size + J->last_page_len[b] : 0;
    if (L > m) m = L;
  }
  return m;
}

static void *worker(void *arg) {
  job_t *J = (job_t *)arg;
  int64_t Lmax = max_len(J);
  double *s = (double *)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
  double *q = (double *)malloc(sizeof(double) * 2 * (size_t)J->head_dim);
  if (!s || !q) {
    pthread_mutex_lock(&J->lock);
    J->error = 1;
    pthread_mutex_unlock(&J->lock);
    free(s);
    free(q);
    return NULL;
  }
  for (;;) {
    pthread_mutex_lock(&J->lock);
    int64_t i = J->next++;
    pthread_mutex_unlock(&J->lock);
    if (i >= J->n_rows) break;
    int64_t r = J->rows ? J->rows[i] : i;
    one_row(J, r, i, s, q);
  }
  free(s);
  free(q);
  return NULL;
}

/*
 * Attention rows r = b * Hq + hq listed in rows[0..n_rows) (rows == NULL:
 * all B * Hq rows in order).  out_o is [n_rows, D] fp64, out_lse [n_rows].
 * dtype (of q, and of the pools when kv_fmt < 0): 0 = fp16, 1 = bf16.
 * kv_fmt: -1 = 16-bit pools; 0 = E4M3 or 1 = E5M2 pools, each value times
 * k_scale (K) or v_scale (V).  rope_theta > 0 turns on rotary positions (an
 * even head_dim is then required).  Returns 0, or 1 on bad arguments / no
 * memory.
 */
int oracle_paged_decode_kv(const uint16_t *q, const void *k_pool, const void *v_pool,
                           const int32_t *kv_indptr, const int32_t *kv_indices,
                           const int32_t *last_page_len, int32_t batch, int32_t num_qo_heads,
                           int32_t num_kv_heads, int32_t head_dim, int32_t page_size,
                           int32_t dtype, int32_t kv_fmt, double sm_scale, double k_scale,
                           double v_scale, double rope_theta, const int64_t *rows,
                           int64_t n_rows, double *out_o, double *out_lse, int32_t n_threads) {
  if (batch < 0 || num_kv_heads <= 0 || num_qo_heads % num_kv_heads || head_dim <= 0 ||
      page_size <= 0 || kv_fmt < -1 || kv_fmt > 1 || (rope_theta > 0.0 && head_dim % 2))
    return 1;
  job_t J;
  memset(&J, 0, sizeof J);
  J.q = q;
  J.k_pool = k_pool;
  J.v_pool = v_pool;
  J.kv_indptr = kv_indptr;
  J.kv_indices = kv_indices;
  J.last_page_len = last_page_len;
  J.batch = batch;
  J.num_qo_heads = num_qo_heads;
  J.num_kv_heads = num_kv_heads;
  J.head_dim = head_dim;
  J.page_size = page_size;
  J.dtype = dtype;
  J.kv_fmt = kv_fmt;
  J.sm_scale = sm_scale;
  J.k_scale = k_scale;
  J.v_scale = v_scale;
  J.rope_theta = rope_theta;
  J.rows = rows;
  J.n_rows = rows ? n_rows : (int64_t)batch * num_qo_heads;
  J.out_o = out_o;
  J.out_lse = out_lse;
  pthread_mutex_init(&J.lock, NULL);
  if (n_threads < 1) n_threads = 1;
  if (n_threads > 256) n_threads = 256;
  pthread_t th[256];
  int started = 0;
  for (int i = 1; i < n_threads; ++i)
    if (pthread_create(&th[started], NULL, worker, &J) == 0) ++started;
  worker(&J);
  for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  pthread_mutex_destroy(&J.lock);
  return J.error;
}

/* The 16-bit decode above with both pools in q's dtype. */
int oracle_paged_decode(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                        const int32_t *kv_indptr, const int32_t *kv_indices,
                        const int32_t *last_page_len, int32_t batch, int32_t num_qo_heads,
                        int32_t num_kv_heads, int32_t head_dim, int32_t page_size,
                        int32_t dtype, double sm_scale, const int64_t *rows, int64_t n_rows,
                        double *out_o, double *out_lse, int32_t n_threads) {
  return oracle_paged_decode_kv(q, k_pool, v_pool, kv_indptr, kv_indices, last_page_len, batch,
                                num_qo_heads, num_kv_heads, head_dim, page_size, dtype, -1,
                                sm_scale, 1.0, 1.0, 0.0, rows, n_rows, out_o, out_lse,
                                n_threads);
}
