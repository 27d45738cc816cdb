/*
 * oracle.c -- fp64 CPU oracle for batched decode attention over a paged
 * KV cache, for the page-append scatter, and for the merge of partial
 * attention states.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load or call this code.  The CUDA
 * library never links, includes or calls it, and it shares no source with
 * the CUDA library: the two meet only through the seeded inputs.
 *
 * What it computes (every function below cites the passage it follows):
 *
 *   decode: for request b and query head h, the exact single-row attention
 *     o = softmax(scale * q K^T) V,   lse = log(sum_t exp(scale * q.k_t)),
 *     with K, V the request's cached keys/values gathered in logical order
 *     through the page table.  This is the standard attention formula
 *     Attention(Q,K,V) = softmax(QK^T/sqrt(d))V ("大模型推理极致优化：
 *     FlashAttention+PageAttention联合调优", section 2.1) restricted to one
 *     query row; FlashAttention is stated there (section 1 and 2.2) to be
 *     mathematically equivalent to it, so the oracle is the definition
 *     written out, not the tiled algorithm.
 *
 *   append: the integer scatter of new tokens into the page slots their
 *     logical positions map to (page = position / page_size through the
 *     page table, "Flash Attention与Paged KV Cache优化大模型推理实战",
 *     section 3.2, and on-demand page allocation, "大模型推理极致优化：
 *     FlashAttention+PageAttention联合调优", section 3.2).
 *
 *   merge: combining attention states of disjoint key sets by their
 *     log-sum-exp weights -- the exact form of the blockwise combination
 *     that "大模型长上下文窗口工程化实战：从RoPE扩展到百万Token推理的生产级部署"
 *     section 4.2 sketches (that sketch averages per-block softmax
 *     outputs, which is not exact; this oracle uses the exact weights).
 *
 *   fp8 KV cache: the same decode and append over a pool of E4M3 codes
 *     ("fp8_e4m3" KV cache of the serving configurations in "上下文窗口优化实战：
 *     如何用PagedAttention+FlashInfer将Llama3-70B的128K上下文吞吐提升3.8倍？"
 *     section 4.1); a key element is code_value * k_scale, a value element
 *     code_value * v_scale, and append stores e4m3(float(x) / scale), round to
 *     nearest even, saturating at +-448.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - pool layout pool[page][K=0|V=1][kv_head][slot][dim], one pool per layer;
 *   - query head h reads KV head h / (Hq/Hkv) (consecutive query heads share);
 *   - page table in CSR form: page_indptr[B+1], page_indices[], and
 *     last_page_len[B]; request b holds (np-1)*page_size + last_page_len[b]
 *     tokens when it owns np > 0 pages, and 0 tokens otherwise;
 *   - a request with no tokens yields o = 0 and lse = -inf;
 *   - lse is the natural-log log-sum-exp of the scaled scores;
 *   - fp8: one binary32 scale for all of K and one for all of V (per-tensor),
 *     the query stays 16-bit, and quantisation divides in binary32 first.
 *
 * Precision: the 16-bit stored values (fp16 or bf16) are widened to double
 * exactly; all arithmetic is in double.  Slots past a request's length are
 * never read (they may hold anything, including NaN).
 *
 * Parallelism: OpenMP over independent (request, head) rows only; each row
 * is computed by one thread in a fixed order, so results do not depend on
 * the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F16 = 0, ORACLE_BF16 = 1, ORACLE_FP8_E4M3 = 3, ORACLE_FP8_E5M2 = 4 };

/* Status codes: 0 ok, otherwise the table or arguments break an invariant
 * that the pages state (valid length within a page, page ids inside the
 * pool: "Flash Attention与Paged KV Cache优化大模型推理实战", section 6.2). */
enum {
  ORACLE_OK = 0,
  ORACLE_BAD_ARG = 1,
  ORACLE_BAD_INDPTR = 2,
  ORACLE_BAD_LAST_LEN = 3,
  ORACLE_BAD_PAGE_ID = 4,
  ORACLE_BAD_APPEND = 5,
  ORACLE_NO_MEMORY = 6
};

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Exact widening of a stored bf16 value: bf16 is the top half of an IEEE
 * binary32, so shifting it into the high bits gives the same number. */
static double widen_bf16(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Exact widening of a stored IEEE binary16 value, from its definition:
 * sign, 5-bit exponent with bias 15, 10-bit fraction, subnormals at e=0. */
static double widen_f16(uint16_t bits) {
  int sign = (bits >> 15) & 1;
  int e = (bits >> 10) & 0x1f;
  int frac = bits & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)frac, -24);               /* frac * 2^-10 * 2^-14 */
  } else if (e == 31) {
    v = frac ? NAN : INFINITY;
  } else {
    v = ldexp((double)(frac | 0x400), e - 25);  /* (1 + frac/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

static double widen(uint16_t bits, int dtype) {
  return dtype == ORACLE_BF16 ? widen_bf16(bits) : widen_f16(bits);
}

/*
 * FP8 E4M3 ("e4m3fn"): sign, 4-bit exponent with bias 7, 3-bit fraction;
 * e = 0 is subnormal (fraction * 2^-9); the code S.1111.111 is NaN and there
 * is no infinity, so the largest finite magnitude is 1.75 * 2^8 = 448.  This
 * is the 8-bit KV-cache format ("fp8_e4m3" in the serving configurations of
 * "上下文窗口优化实战：如何用PagedAttention+FlashInfer将Llama3-70B的128K上下文吞吐提升3.8倍？"
 * section 4.1 and "大模型长上下文窗口工程化实战：从RoPE扩展到百万Token推理的生产级部署"
 * section 3.2); a stored code means code_value * scale, one scale for all K and
 * one for all V.
 */
static double widen_e4m3(uint8_t code) {
  const int sign = code >> 7, e = (code >> 3) & 0xf, frac = code & 7;
  double v;
  if (e == 15 && frac == 7) return NAN;
  if (e == 0) v = ldexp((double)frac, -9);
  else v = ldexp((double)(frac | 8), e - 10);  /* (1 + frac/8) * 2^(e-7) */
  return sign ? -v : v;
}

int oracle_e4m3_decode(const uint8_t* codes, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = widen_e4m3(codes[i]);
  return ORACLE_OK;
}

/*
 * Encode x / scale (both binary32; the quotient rounded once to binary32) as
 * E4M3: round to the nearest representable value, ties to the even code;
 * magnitudes beyond 448 saturate to +-448; NaN stays NaN.  The nearest value
 * is found by comparing against every finite code -- slow, and plainly the
 * definition.
 */
static uint8_t encode_e4m3(float x, float scale) {
  const float q = x / scale;
  if (isnan(q)) return 0x7f;
  const double v = (double)q;
  const int neg = signbit(q) ? 1 : 0;
  const double a = fabs(v);
  if (a >= 448.0) return (uint8_t)((neg << 7) | 0x7e);
  int best = 0;
  double best_err = INFINITY;
  for (int c = 0; c < 0x7f; ++c) {           /* non-negative finite codes */
    const double err = fabs(widen_e4m3((uint8_t)c) - a);
    if (err < best_err || (err == best_err && (c & 1) == 0)) {
      best = c;
      best_err = err;
    }
  }
  return (uint8_t)((neg << 7) | best);
}

int oracle_e4m3_encode(const float* x, int64_t n, float scale, uint8_t* codes) {
  if (!(scale > 0.0f) || isinf(scale)) return ORACLE_BAD_ARG;
  for (int64_t i = 0; i < n; ++i) codes[i] = encode_e4m3(x[i], scale);
  return ORACLE_OK;
}

/*
 * FP8 E5M2: sign, 5-bit exponent with bias 15, 2-bit fraction -- the top
 * byte of an IEEE half, so it keeps infinities (S.11111.00) and NaNs
 * (S.11111.xx, xx != 0); largest finite magnitude 1.75 * 2^15 = 57344.  The
 * "fp8_e5m2" KV-cache dtype of "大模型长上下文窗口工程化实战：从RoPE扩展到百万
 * Token推理的生产级部署" sections 3.1 and 3.2; scales as for E4M3.
 */
static double widen_e5m2(uint8_t code) {
  const int sign = code >> 7, e = (code >> 2) & 0x1f, frac = code & 3;
  double v;
  if (e == 31) v = frac ? NAN : INFINITY;
  else if (e == 0) v = ldexp((double)frac, -16);      /* frac/4 * 2^-14 */
  else v = ldexp((double)(frac | 4), e - 17);         /* (1 + frac/4) * 2^(e-15) */
  return sign ? -v : v;
}

int oracle_e5m2_decode(const uint8_t* codes, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = widen_e5m2(codes[i]);
  return ORACLE_OK;
}

/* x / scale as E5M2: nearest finite value, ties to the even code, magnitudes
 * from 57344 up (infinity included) saturating to +-57344, NaN to 0x7f. */
static uint8_t encode_e5m2(float x, float scale) {
  const float q = (float)(x / scale);  /* binary32 quotient */
  if (isnan(q)) return 0x7f;
  const int neg = signbit(q) ? 1 : 0;
  const double a = fabs((double)q);
  if (a >= 57344.0) return (uint8_t)((neg << 7) | 0x7b);
  int best = 0;
  double best_err = INFINITY;
  for (int c = 0; c <= 0x7b; ++c) {          /* non-negative finite codes */
    const double err = fabs(widen_e5m2((uint8_t)c) - a);
    if (err < best_err || (err == best_err && !(c & 1))) {     /* tie: even code */
      best = c;
      best_err = err;
    }
  }
  return (uint8_t)((neg << 7) | best);
}

int oracle_e5m2_encode(const float* x, int64_t n, float scale, uint8_t* codes) {
  if (!(scale > 0.0f) || isinf(scale)) return ORACLE_BAD_ARG;
  for (int64_t i = 0; i < n; ++i) codes[i] = encode_e5m2(x[i], scale);
  return ORACLE_OK;
}

static int is_fp8(int dtype) { return dtype == ORACLE_FP8_E4M3 || dtype == ORACLE_FP8_E5M2; }

/* Element idx of a pool of 16-bit (fp16 / bf16) or 8-bit (E4M3 / E5M2) values,
 * widened exactly (8-bit codes are multiplied by their scale afterwards). */
static double kv_elem(const void* pool, int kv_dtype, size_t idx) {
  if (kv_dtype == ORACLE_FP8_E4M3) return widen_e4m3(((const uint8_t*)pool)[idx]);
  if (kv_dtype == ORACLE_FP8_E5M2) return widen_e5m2(((const uint8_t*)pool)[idx]);
  return widen(((const uint16_t*)pool)[idx], kv_dtype);
}

/* Tokens held by request b under the CSR page table.  Returns -1 when the
 * table breaks an invariant. */
static int64_t request_len(int b, int page_size, const int32_t* page_indptr,
                           const int32_t* last_page_len, int* why) {
  int64_t np = (int64_t)page_indptr[b + 1] - (int64_t)page_indptr[b];
  if (page_indptr[b] < 0 || np < 0) { *why = ORACLE_BAD_INDPTR; return -1; }
  if (np == 0) return 0;
  if (last_page_len[b] < 1 || last_page_len[b] > page_size) {
    *why = ORACLE_BAD_LAST_LEN;
    return -1;
  }
  return (np - 1) * (int64_t)page_size + last_page_len[b];
}

/* Element offset of (page, kv, head, slot, dim 0) in the pool. */
static size_t pool_offset(int64_t page, int kv, int head, int64_t slot,
                          int num_kv_heads, int page_size, int head_dim) {
  return ((((size_t)page * 2 + (size_t)kv) * (size_t)num_kv_heads + (size_t)head) *
              (size_t)page_size + (size_t)slot) * (size_t)head_dim;
}

/* Validate the whole table once (so worker threads never fail midway). */
static int check_table(int64_t num_pages, int page_size, int batch,
                       const int32_t* page_indptr, const int32_t* page_indices,
                       const int32_t* last_page_len) {
  for (int b = 0; b < batch; ++b) {
    int why = ORACLE_OK;
    if (request_len(b, page_size, page_indptr, last_page_len, &why) < 0) return why;
    for (int32_t i = page_indptr[b]; i < page_indptr[b + 1]; ++i) {
      if (page_indices[i] < 0 || (int64_t)page_indices[i] >= num_pages) return ORACLE_BAD_PAGE_ID;
    }
  }
  return ORACLE_OK;
}

/*
 * oracle_decode -- exact decode attention, one query token per request.
 *
 * q        [batch][num_qo_heads][head_dim]   16-bit stored values
 * pool     [num_pages][2][num_kv_heads][page_size][head_dim]   16-bit
 * out      [batch][num_qo_heads][head_dim]   double, written
 * lse      [batch][num_qo_heads]             double, written (natural log)
 *
 * For each (b, h): s_t = scale * sum_d q[d] K[t][d]; m = max_t s_t;
 * l = sum_t exp(s_t - m); o[d] = sum_t exp(s_t - m) V[t][d] / l;
 * lse = m + log(l).  Subtracting m changes nothing mathematically (the
 * factor exp(-m) cancels between numerator and l); it only keeps exp()
 * in range.
 */
static int decode_rows(const uint16_t* q, int q_dtype, const void* pool, int kv_dtype,
                       double k_scale, double v_scale,
                       int64_t num_pages, int page_size, int num_kv_heads, int head_dim,
                       int batch, int num_qo_heads,
                       const int32_t* page_indptr, const int32_t* page_indices,
                       const int32_t* last_page_len, double scale,
                       double* out, double* lse) {
  if (batch < 0 || page_size < 1 || num_kv_heads < 1 || head_dim < 1 ||
      num_qo_heads < num_kv_heads || num_qo_heads % num_kv_heads != 0 ||
      (q_dtype != ORACLE_F16 && q_dtype != ORACLE_BF16) ||
      (kv_dtype != ORACLE_F16 && kv_dtype != ORACLE_BF16 && !is_fp8(kv_dtype)))
    return ORACLE_BAD_ARG;
  int rc = check_table(num_pages, page_size, batch, page_indptr, page_indices, last_page_len);
  if (rc != ORACLE_OK) return rc;
  const int group = num_qo_heads / num_kv_heads;
  const int64_t rows = (int64_t)batch * num_qo_heads;
  int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t row = 0; row < rows; ++row) {
    const int b = (int)(row / num_qo_heads);
    const int h = (int)(row % num_qo_heads);
    const int g = h / group;
    int why = ORACLE_OK;
    const int64_t len = request_len(b, page_size, page_indptr, last_page_len, &why);
    double* o = out + (size_t)row * head_dim;
    if (len == 0) {
      for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
      lse[row] = -INFINITY;
      continue;
    }
    double* qd = (double*)malloc(sizeof(double) * (size_t)head_dim);
    double* s = (double*)malloc(sizeof(double) * (size_t)len);
    if (!qd || !s) {
      free(qd); free(s);
#pragma omp atomic write
      failed = 1;
      continue;
    }
    for (int d = 0; d < head_dim; ++d) qd[d] = widen(q[(size_t)row * head_dim + d], q_dtype);

    /* scores, in logical token order */
    for (int64_t t = 0; t < len; ++t) {
      const int64_t page = page_indices[page_indptr[b] + t / page_size];
      const size_t k = pool_offset(page, 0, g, t % page_size,
                                   num_kv_heads, page_size, head_dim);
      double dot = 0.0;
      for (int d = 0; d < head_dim; ++d) dot += qd[d] * (kv_elem(pool, kv_dtype, k + d) * k_scale);
      s[t] = scale * dot;
    }
    double m = -INFINITY;
    for (int64_t t = 0; t < len; ++t) if (s[t] > m) m = s[t];

    double l = 0.0;
    for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
    for (int64_t t = 0; t < len; ++t) {
      const double w = exp(s[t] - m);
      const int64_t page = page_indices[page_indptr[b] + t / page_size];
      const size_t v = pool_offset(page, 1, g, t % page_size,
                                   num_kv_heads, page_size, head_dim);
      l += w;
      for (int d = 0; d < head_dim; ++d) o[d] += w * (kv_elem(pool, kv_dtype, v + d) * v_scale);
    }
    for (int d = 0; d < head_dim; ++d) o[d] /= l;
    lse[row] = m + log(l);
    free(qd);
    free(s);
  }
  return failed ? ORACLE_NO_MEMORY : ORACLE_OK;
}

int oracle_decode(const uint16_t* q, const uint16_t* pool, int dtype,
                  int64_t num_pages, int page_size, int num_kv_heads, int head_dim,
                  int batch, int num_qo_heads,
                  const int32_t* page_indptr, const int32_t* page_indices,
                  const int32_t* last_page_len, double scale,
                  double* out, double* lse) {
  if (is_fp8(dtype)) return ORACLE_BAD_ARG;
  return decode_rows(q, dtype, pool, dtype, 1.0, 1.0, num_pages, page_size, num_kv_heads,
                     head_dim, batch, num_qo_heads, page_indptr, page_indices, last_page_len,
                     scale, out, lse);
}

/*
 * oracle_decode_fp8 -- the same attention over an 8-bit pool (fp8_dtype
 * ORACLE_FP8_E4M3 or ORACLE_FP8_E5M2): key element = code_value * k_scale,
 * value element = code_value * v_scale (exact in double); q is fp16 or bf16
 * (q_dtype).
 */
int oracle_decode_fp8(const uint16_t* q, int q_dtype, const uint8_t* pool, int fp8_dtype,
                      float k_scale, float v_scale, int64_t num_pages, int page_size,
                      int num_kv_heads, int head_dim, int batch, int num_qo_heads,
                      const int32_t* page_indptr, const int32_t* page_indices,
                      const int32_t* last_page_len, double scale, double* out, double* lse) {
  if (!is_fp8(fp8_dtype)) return ORACLE_BAD_ARG;
  return decode_rows(q, q_dtype, pool, fp8_dtype, (double)k_scale, (double)v_scale,
                     num_pages, page_size, num_kv_heads, head_dim, batch, num_qo_heads,
                     page_indptr, page_indices, last_page_len, scale, out, lse);
}

/*
 * oracle_append -- scatter new tokens into their pages (in place).
 *
 * The table passed is the table AFTER the append: the caller has already
 * allocated any page the new tokens need.  Request b appends the
 * n_b = append_indptr[b+1] - append_indptr[b] rows
 * k_new/v_new[append_indptr[b] + i] (i < n_b, each [num_kv_heads][head_dim])
 * at logical positions len_b - n_b + i, where len_b is its length after the
 * append.  Position p lives in page page_indices[page_indptr[b] + p / page_size]
 * at slot p % page_size.  Pure copies of the 16-bit patterns; every other
 * byte of the pool is left as it was.
 */
static int append_rows(void* pool, int kv_dtype, float k_scale, float v_scale,
                       int64_t num_pages, int page_size, int num_kv_heads,
                       int head_dim, int batch,
                       const int32_t* page_indptr, const int32_t* page_indices,
                       const int32_t* last_page_len,
                       const uint16_t* k_new, const uint16_t* v_new, int new_dtype,
                       const int32_t* append_indptr) {
  if (batch < 0 || page_size < 1 || num_kv_heads < 1 || head_dim < 1) return ORACLE_BAD_ARG;
  if (!is_fp8(kv_dtype) && kv_dtype != new_dtype) return ORACLE_BAD_ARG;
  int rc = check_table(num_pages, page_size, batch, page_indptr, page_indices, last_page_len);
  if (rc != ORACLE_OK) return rc;
  if (append_indptr[0] < 0) return ORACLE_BAD_APPEND;
  for (int b = 0; b < batch; ++b) {
    int why = ORACLE_OK;
    const int64_t len = request_len(b, page_size, page_indptr, last_page_len, &why);
    const int64_t n_new = (int64_t)append_indptr[b + 1] - append_indptr[b];
    if (n_new < 0 || n_new > len) return ORACLE_BAD_APPEND;
  }
  const size_t row = (size_t)num_kv_heads * (size_t)head_dim;
  for (int b = 0; b < batch; ++b) {
    int why = ORACLE_OK;
    const int64_t len = request_len(b, page_size, page_indptr, last_page_len, &why);
    const int64_t n_new = (int64_t)append_indptr[b + 1] - append_indptr[b];
    for (int64_t i = 0; i < n_new; ++i) {
      const int64_t pos = len - n_new + i;
      const int64_t page = page_indices[page_indptr[b] + pos / page_size];
      const int64_t slot = pos % page_size;
      const size_t src = ((size_t)append_indptr[b] + (size_t)i) * row;
      for (int h = 0; h < num_kv_heads; ++h) {
        const size_t dk = pool_offset(page, 0, h, slot, num_kv_heads, page_size, head_dim);
        const size_t dv = pool_offset(page, 1, h, slot, num_kv_heads, page_size, head_dim);
        const uint16_t* ks = k_new + src + (size_t)h * head_dim;
        const uint16_t* vs = v_new + src + (size_t)h * head_dim;
        if (kv_dtype == ORACLE_FP8_E4M3) {
          /* quantise: the 16-bit value widened to binary32, divided by the scale */
          uint8_t* p8 = (uint8_t*)pool;
          for (int d = 0; d < head_dim; ++d) {
            p8[dk + d] = encode_e4m3((float)widen(ks[d], new_dtype), k_scale);
            p8[dv + d] = encode_e4m3((float)widen(vs[d], new_dtype), v_scale);
          }
        } else if (kv_dtype == ORACLE_FP8_E5M2) {
          uint8_t* p8 = (uint8_t*)pool;
          for (int d = 0; d < head_dim; ++d) {
            p8[dk + d] = encode_e5m2((float)widen(ks[d], new_dtype), k_scale);
            p8[dv + d] = encode_e5m2((float)widen(vs[d], new_dtype), v_scale);
          }
        } else {
          memcpy((uint16_t*)pool + dk, ks, sizeof(uint16_t) * (size_t)head_dim);
          memcpy((uint16_t*)pool + dv, vs, sizeof(uint16_t) * (size_t)head_dim);
        }
      }
    }
  }
  return ORACLE_OK;
}

int oracle_append(uint16_t* pool, int64_t num_pages, int page_size, int num_kv_heads,
                  int head_dim, int batch,
                  const int32_t* page_indptr, const int32_t* page_indices,
                  const int32_t* last_page_len,
                  const uint16_t* k_new, const uint16_t* v_new,
                  const int32_t* append_indptr) {
  /* the 16-bit type is irrelevant to a bit copy; BF16 stands for either */
  return append_rows(pool, ORACLE_BF16, 1.0f, 1.0f, num_pages, page_size, num_kv_heads,
                     head_dim, batch, page_indptr, page_indices, last_page_len, k_new, v_new,
                     ORACLE_BF16, append_indptr);
}

/*
 * oracle_append_fp8 -- the same scatter into an 8-bit pool (fp8_dtype): every
 * new element is quantised as encode(value / scale) (k_scale for K, v_scale
 * for V).
 */
int oracle_append_fp8(uint8_t* pool, int fp8_dtype, float k_scale, float v_scale,
                      int64_t num_pages, int page_size, int num_kv_heads, int head_dim, int batch,
                      const int32_t* page_indptr, const int32_t* page_indices,
                      const int32_t* last_page_len, const uint16_t* k_new,
                      const uint16_t* v_new, int new_dtype, const int32_t* append_indptr) {
  if (!(k_scale > 0.0f) || !(v_scale > 0.0f) || isinf(k_scale) || isinf(v_scale))
    return ORACLE_BAD_ARG;
  if (new_dtype != ORACLE_F16 && new_dtype != ORACLE_BF16) return ORACLE_BAD_ARG;
  if (!is_fp8(fp8_dtype)) return ORACLE_BAD_ARG;
  return append_rows(pool, fp8_dtype, k_scale, v_scale, num_pages, page_size,
                     num_kv_heads, head_dim, batch, page_indptr, page_indices, last_page_len,
                     k_new, v_new, new_dtype, append_indptr);
}

/*
 * Visibility of key position t to a query at position pos in a chunk of new
 * tokens: causal (t <= pos: the cache holds nothing later), and with a
 * window (window_left >= 0) also within window_left positions before the
 * query, or when the key is one of the first sink_tokens positions.  This is
 * the window-plus-global-tokens mask of "大模型长上下文窗口工程化实战：从RoPE扩展到
 * 百万Token推理的生产级部署" section 2.3 (half-width window_size / 2 on each
 * side, global tokens seeing and seen by everything) with its right half cut
 * off by causality; its rule that global queries see every key adds nothing
 * then, since every key such a query may see is itself a global token.
 */
static int key_visible(int64_t t, int64_t pos, int window_left, int sink_tokens) {
  if (t > pos) return 0;
  if (window_left < 0) return 1;
  return t >= pos - window_left || t < sink_tokens;
}

/*
 * oracle_append_attention -- exact attention of a chunk of new query tokens
 * per request over the paged cache (chunked prefill: a prompt processed a
 * chunk at a time against the cache that already holds the earlier chunks,
 * "大模型长上下文窗口工程化实战：从RoPE扩展到百万Token推理的生产级部署" section 3.1;
 * also several speculative tokens verified at once).
 *
 * q         [nnz_q][num_qo_heads][head_dim] 16-bit; request b's query tokens
 *           are rows qo_indptr[b] .. qo_indptr[b+1]-1 (qo_indptr[0] = 0,
 *           nnz_q = qo_indptr[batch])
 * table     the table after the chunk's K/V were appended: request b holds
 *           L_b tokens and its q_len_b = qo_indptr[b+1] - qo_indptr[b] query
 *           tokens are the last q_len_b of them, so query i is at position
 *           pos = L_b - q_len_b + i
 * out, lse  [nnz_q][num_qo_heads][head_dim] and [nnz_q][num_qo_heads]
 *
 * For each (query row, head h): the single-row attention of the decode over
 * the keys t with key_visible(t, pos); GQA as in the decode.  Every query
 * sees at least its own key.
 */
int oracle_append_attention(const uint16_t* q, const uint16_t* pool, int dtype,
                            int64_t num_pages, int page_size, int num_kv_heads, int head_dim,
                            int batch, int num_qo_heads,
                            const int32_t* page_indptr, const int32_t* page_indices,
                            const int32_t* last_page_len, const int32_t* qo_indptr,
                            int window_left, int sink_tokens, double scale,
                            double* out, double* lse) {
  if (batch < 0 || page_size < 1 || num_kv_heads < 1 || head_dim < 1 ||
      num_qo_heads < num_kv_heads || num_qo_heads % num_kv_heads != 0 || sink_tokens < 0 ||
      (dtype != ORACLE_F16 && dtype != ORACLE_BF16))
    return ORACLE_BAD_ARG;
  int rc = check_table(num_pages, page_size, batch, page_indptr, page_indices, last_page_len);
  if (rc != ORACLE_OK) return rc;
  if (batch > 0 && qo_indptr[0] != 0) return ORACLE_BAD_APPEND;
  for (int b = 0; b < batch; ++b) {
    int why = ORACLE_OK;
    const int64_t len = request_len(b, page_size, page_indptr, last_page_len, &why);
    const int64_t n_q = (int64_t)qo_indptr[b + 1] - qo_indptr[b];
    if (n_q < 0 || n_q > len) return ORACLE_BAD_APPEND;
  }
  const int64_t nnz = batch > 0 ? (int64_t)qo_indptr[batch] : 0;
  /* request of every query row */
  int* req = (int*)malloc(sizeof(int) * (size_t)(nnz > 0 ? nnz : 1));
  if (!req) return ORACLE_NO_MEMORY;
  for (int b = 0; b < batch; ++b)
    for (int64_t r = qo_indptr[b]; r < qo_indptr[b + 1]; ++r) req[r] = b;
  const int group = num_qo_heads / num_kv_heads;
  int failed = 0;

#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t row = 0; row < nnz * num_qo_heads; ++row) {
    const int64_t r = row / num_qo_heads;    /* query token */
    const int h = (int)(row % num_qo_heads);
    const int b = req[r];
    const int kvh = h / group;
    int why = ORACLE_OK;
    const int64_t len = request_len(b, page_size, page_indptr, last_page_len, &why);
    const int64_t n_q = (int64_t)qo_indptr[b + 1] - qo_indptr[b];
    const int64_t pos = len - n_q + (r - qo_indptr[b]);
    double* o = out + (size_t)row * head_dim;
    double* qd = (double*)malloc(sizeof(double) * (size_t)head_dim);
    double* s = (double*)malloc(sizeof(double) * (size_t)(pos + 1));
    if (!qd || !s) {
      free(qd); free(s);
#pragma omp atomic write
      failed = 1;
      continue;
    }
    for (int d = 0; d < head_dim; ++d) qd[d] = widen(q[(size_t)row * head_dim + d], dtype);
    double m = -INFINITY;
    for (int64_t t = 0; t <= pos; ++t) {
      if (!key_visible(t, pos, window_left, sink_tokens)) { s[t] = -INFINITY; continue; }
      const int64_t page = page_indices[page_indptr[b] + t / page_size];
      const size_t kk = pool_offset(page, 0, kvh, t % page_size, num_kv_heads, page_size, head_dim);
      double dot = 0.0;
      for (int d = 0; d < head_dim; ++d) dot += qd[d] * widen(pool[kk + d], dtype);
      s[t] = dot * scale;
      if (s[t] > m) m = s[t];
    }
    double l = 0.0;
    for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
    for (int64_t t = 0; t <= pos; ++t) {
      if (s[t] == -INFINITY) continue;          /* invisible: weight exactly 0 */
      const double wt = exp(s[t] - m);
      const int64_t page = page_indices[page_indptr[b] + t / page_size];
      const size_t vv = pool_offset(page, 1, kvh, t % page_size, num_kv_heads, page_size, head_dim);
      l += wt;
      for (int d = 0; d < head_dim; ++d) o[d] += wt * widen(pool[vv + d], dtype);
    }
    for (int d = 0; d < head_dim; ++d) o[d] /= l;
    lse[row] = log(l) + m;
    free(qd);
    free(s);
  }
  free(req);
  return failed ? ORACLE_NO_MEMORY : ORACLE_OK;
}

/*
 * oracle_merge -- combine S attention states per (row, head).
 *
 * v [rows][S][H][D] are normalised partial outputs, s [rows][S][H] their
 * natural-log log-sum-exp values.  With M = max_j s_j and w_j = exp(s_j - M):
 *   v_out = sum_j w_j v_j / sum_j w_j,   s_out = M + log(sum_j w_j).
 * A state with s = -inf has weight 0; if every state has s = -inf the
 * result is v_out = 0, s_out = -inf (the value of attention over no keys).
 */
void oracle_merge(const double* v, const double* s, int64_t rows, int num_states,
                  int num_heads, int head_dim, double* v_out, double* s_out) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int h = 0; h < num_heads; ++h) {
      double m = -INFINITY;
      for (int j = 0; j < num_states; ++j) {
        const double sj = s[((size_t)r * num_states + j) * num_heads + h];
        if (sj > m) m = sj;
      }
      double* o = v_out + ((size_t)r * num_heads + h) * head_dim;
      for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
      if (m == -INFINITY) {
        s_out[(size_t)r * num_heads + h] = -INFINITY;
        continue;
      }
      double wsum = 0.0;
      for (int j = 0; j < num_states; ++j) {
        const double sj = s[((size_t)r * num_states + j) * num_heads + h];
        if (sj == -INFINITY) continue;           /* weight exactly 0 */
        const double w = exp(sj - m);
        const double* vj = v + (((size_t)r * num_states + j) * num_heads + h) * head_dim;
        wsum += w;
        for (int d = 0; d < head_dim; ++d) o[d] += w * vj[d];
      }
      for (int d = 0; d < head_dim; ++d) o[d] /= wsum;
      s_out[(size_t)r * num_heads + h] = m + log(wsum);
    }
  }
}
