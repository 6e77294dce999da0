/*
 * oracle.c -- FP64, single-threaded definition of paged quantised-KV GQA
 * attention.  TEST INFRASTRUCTURE ONLY (see oracle.h): the product library
 * never includes or links this file.
 *
 * Written from the formula out = softmax(scale * Q * dequant(K)^T + mask) *
 * dequant(V) and the cache description of the INT4 paged-KV page
 * (onnxruntime PR 32515, Code analysis 2 and 3).  Readings of points the pages
 * leave open are stated beside the code that depends on them.
 */
#include "oracle.h"

#include <math.h>
#include <stddef.h>
#include <stdlib.h>

int oracle_cache_head_size(int kv_dtype, int head_size) {
  /* INT4-KV page, Code analysis 2: (head_size + 1) / 2 for packed INT4. */
  if (kv_dtype == ORACLE_KV_INT4) return (head_size + 1) / 2;
  return head_size;
}

/* OCP 8-bit floating point, E4M3 "fn" variant: 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits; exponent field 0 is subnormal; the all-ones
 * exponent is an ordinary binade except mantissa 7, which is NaN. */
static double decode_e4m3(uint8_t c) {
  int sign = (c >> 7) & 1;
  int e = (c >> 3) & 0xF;
  int m = c & 0x7;
  double v;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0)
    v = ldexp((double)m / 8.0, 1 - 7);
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

double oracle_decode(int kv_dtype, const uint8_t* row, int d) {
  if (kv_dtype == ORACLE_KV_INT8) return (double)(int8_t)row[d];
  if (kv_dtype == ORACLE_KV_INT4) {
    /* Reading (pages silent on order and sign): channel 2j is the low nibble
     * of byte j, channel 2j+1 the high nibble; two's complement in [-8, 7]. */
    uint8_t byte = row[d / 2];
    int nib = (d % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    return (double)(nib >= 8 ? nib - 16 : nib);
  }
  return decode_e4m3(row[d]);
}

int oracle_pack_int4(const int8_t* src, int64_t rows, int head_size, uint8_t* dst) {
  int chs = (head_size + 1) / 2;
  for (int64_t r = 0; r < rows; ++r) {
    for (int j = 0; j < chs; ++j) {
      int lo = src[r * head_size + 2 * j];
      int hi = (2 * j + 1 < head_size) ? src[r * head_size + 2 * j + 1] : 0;
      if (lo < -8 || lo > 7 || hi < -8 || hi > 7) return ORACLE_EINVAL;
      dst[r * chs + j] = (uint8_t)((lo & 0xF) | ((hi & 0xF) << 4));
    }
  }
  return ORACLE_OK;
}

int oracle_unpack_int4(const uint8_t* src, int64_t rows, int head_size, int8_t* dst) {
  int chs = (head_size + 1) / 2;
  for (int64_t r = 0; r < rows; ++r)
    for (int d = 0; d < head_size; ++d)
      dst[r * head_size + d] = (int8_t)oracle_decode(ORACLE_KV_INT4, src + r * chs, d);
  return ORACLE_OK;
}

/* Contract checks shared by the attention entry points.  Reading of the
 * sequence lengths: seqlens_k[b] counts every key in the cache for sequence b,
 * the new tokens included, so the past length is L_b - q_b >= 0. */
static int check_problem(const oracle_problem* p, const int32_t* seqlens_k,
                         const int32_t* cu_seqlens_q) {
  if (p->batch < 0 || p->num_heads <= 0 || p->kv_num_heads <= 0 || p->head_size <= 0 ||
      p->block_size <= 0 || p->num_blocks < 0 || p->max_blocks_per_seq < 0)
    return ORACLE_EINVAL;
  if (p->num_heads % p->kv_num_heads != 0) return ORACLE_EINVAL;
  if (p->kv_dtype < ORACLE_KV_INT8 || p->kv_dtype > ORACLE_KV_FP8_E4M3) return ORACLE_EINVAL;
  if (cu_seqlens_q[0] != 0) return ORACLE_EINVAL;
  for (int b = 0; b < p->batch; ++b) {
    int qb = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
    int Lb = seqlens_k[b];
    if (qb < 0 || Lb < qb) return ORACLE_EINVAL;
    if ((int64_t)Lb > (int64_t)p->max_blocks_per_seq * p->block_size) return ORACLE_EINVAL;
  }
  return ORACLE_OK;
}

static const uint8_t* cache_row(const oracle_problem* p, const uint8_t* cache,
                                const int32_t* block_table, int b, int t, int kv) {
  int chs = oracle_cache_head_size(p->kv_dtype, p->head_size);
  int32_t phys = block_table[(int64_t)b * p->max_blocks_per_seq + t / p->block_size];
  int slot = t % p->block_size;
  return cache + (((int64_t)phys * p->block_size + slot) * p->kv_num_heads + kv) * chs;
}

static int check_block_table(const oracle_problem* p, const int32_t* block_table,
                             const int32_t* seqlens_k) {
  for (int b = 0; b < p->batch; ++b) {
    int nblk = (seqlens_k[b] + p->block_size - 1) / p->block_size;
    for (int l = 0; l < nblk; ++l) {
      int32_t phys = block_table[(int64_t)b * p->max_blocks_per_seq + l];
      if (phys < 0 || phys >= p->num_blocks) return ORACLE_EINVAL;
    }
  }
  return ORACLE_OK;
}

/* Number of keys new token i of sequence b may attend to.  Reading of the
 * causal alignment: bottom-right, new token i sits at absolute position
 * (L_b - q_b) + i and sees keys t <= that position; without the mask every
 * token sees all L_b keys.  For decode (q_b = 1) both give L_b. */
static int visible_keys(const oracle_problem* p, int Lb, int qb, int i) {
  return p->causal ? (Lb - qb) + i + 1 : Lb;
}

static double softmax_scale_of(const oracle_problem* p) {
  return p->softmax_scale != 0.0 ? p->softmax_scale : 1.0 / sqrt((double)p->head_size);
}

int oracle_paged_attn(const oracle_problem* p, const double* q, const uint8_t* k_cache,
                      const uint8_t* v_cache, const double* k_scale, const double* v_scale,
                      const int32_t* block_table, const int32_t* seqlens_k,
                      const int32_t* cu_seqlens_q, double* out) {
  if (check_problem(p, seqlens_k, cu_seqlens_q) != ORACLE_OK) return ORACLE_EINVAL;
  if (check_block_table(p, block_table, seqlens_k) != ORACLE_OK) return ORACLE_EINVAL;
  const int H = p->num_heads, D = p->head_size, G = p->num_heads / p->kv_num_heads;
  const double scale = softmax_scale_of(p);
  int maxL = 0;
  for (int b = 0; b < p->batch; ++b)
    if (seqlens_k[b] > maxL) maxL = seqlens_k[b];
  double* s = (double*)malloc(sizeof(double) * (maxL > 0 ? maxL : 1));
  if (!s) return ORACLE_EINVAL;

  for (int b = 0; b < p->batch; ++b) {
    const int Lb = seqlens_k[b];
    const int qb = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
    for (int i = 0; i < qb; ++i) {
      const int nk = visible_keys(p, Lb, qb, i);
      const int64_t tok = cu_seqlens_q[b] + i;
      for (int h = 0; h < H; ++h) {
        const int kv = h / G; /* reading: contiguous query-head groups */
        const double* qrow = q + (tok * H + h) * D;
        /* logits s_t = scale * sum_d q[d] * k_scale[kv, d] * decode(K)[t, d] */
        double smax = -INFINITY;
        for (int t = 0; t < nk; ++t) {
          const uint8_t* krow = cache_row(p, k_cache, block_table, b, t, kv);
          double acc = 0.0;
          for (int d = 0; d < D; ++d)
            acc += qrow[d] * (k_scale[kv * D + d] * oracle_decode(p->kv_dtype, krow, d));
          s[t] = scale * acc;
          if (s[t] > smax) smax = s[t];
        }
        /* w_t = exp(s_t - max) / sum exp(s_u - max) */
        double denom = 0.0;
        for (int t = 0; t < nk; ++t) {
          s[t] = exp(s[t] - smax);
          denom += s[t];
        }
        double* orow = out + (tok * H + h) * D;
        for (int d = 0; d < D; ++d) orow[d] = 0.0;
        for (int t = 0; t < nk; ++t) {
          const uint8_t* vrow = cache_row(p, v_cache, block_table, b, t, kv);
          const double w = s[t] / denom;
          for (int d = 0; d < D; ++d)
            orow[d] += w * (v_scale[kv * D + d] * oracle_decode(p->kv_dtype, vrow, d));
        }
      }
    }
  }
  free(s);
  return ORACLE_OK;
}

int oracle_paged_attn_folded(const oracle_problem* p, const double* q, const uint8_t* k_cache,
                             const uint8_t* v_cache, const double* k_scale,
                             const double* v_scale, const int32_t* block_table,
                             const int32_t* seqlens_k, const int32_t* cu_seqlens_q,
                             double* out) {
  if (check_problem(p, seqlens_k, cu_seqlens_q) != ORACLE_OK) return ORACLE_EINVAL;
  if (check_block_table(p, block_table, seqlens_k) != ORACLE_OK) return ORACLE_EINVAL;
  const int H = p->num_heads, D = p->head_size, G = p->num_heads / p->kv_num_heads;
  const double scale = softmax_scale_of(p);
  int maxL = 0;
  for (int b = 0; b < p->batch; ++b)
    if (seqlens_k[b] > maxL) maxL = seqlens_k[b];
  double* s = (double*)malloc(sizeof(double) * (maxL > 0 ? maxL : 1));
  double* qf = (double*)malloc(sizeof(double) * D);
  double* acc_v = (double*)malloc(sizeof(double) * D);
  if (!s || !qf || !acc_v) {
    free(s);
    free(qf);
    free(acc_v);
    return ORACLE_EINVAL;
  }
  for (int b = 0; b < p->batch; ++b) {
    const int Lb = seqlens_k[b];
    const int qb = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
    for (int i = 0; i < qb; ++i) {
      const int nk = visible_keys(p, Lb, qb, i);
      const int64_t tok = cu_seqlens_q[b] + i;
      for (int h = 0; h < H; ++h) {
        const int kv = h / G;
        /* Normaliser: 2^e with e the frexp exponent of max_d |k_scale[kv, d]|
         * (INT4-KV page, Code analysis 3); max = 0 gives e = 0. */
        double kmax = 0.0;
        for (int d = 0; d < D; ++d)
          if (fabs(k_scale[kv * D + d]) > kmax) kmax = fabs(k_scale[kv * D + d]);
        int e = 0;
        (void)frexp(kmax, &e);
        const double* qrow = q + (tok * H + h) * D;
        for (int d = 0; d < D; ++d) qf[d] = qrow[d] * ldexp(k_scale[kv * D + d], -e);
        const double c = scale * ldexp(1.0, e);
        double smax = -INFINITY;
        for (int t = 0; t < nk; ++t) {
          const uint8_t* krow = cache_row(p, k_cache, block_table, b, t, kv);
          double acc = 0.0;
          for (int d = 0; d < D; ++d) acc += qf[d] * oracle_decode(p->kv_dtype, krow, d);
          s[t] = c * acc;
          if (s[t] > smax) smax = s[t];
        }
        double denom = 0.0;
        for (int t = 0; t < nk; ++t) {
          s[t] = exp(s[t] - smax);
          denom += s[t];
        }
        for (int d = 0; d < D; ++d) acc_v[d] = 0.0;
        for (int t = 0; t < nk; ++t) {
          const uint8_t* vrow = cache_row(p, v_cache, block_table, b, t, kv);
          for (int d = 0; d < D; ++d) acc_v[d] += s[t] * oracle_decode(p->kv_dtype, vrow, d);
        }
        double* orow = out + (tok * H + h) * D;
        for (int d = 0; d < D; ++d) orow[d] = v_scale[kv * D + d] * acc_v[d] / denom;
      }
    }
  }
  free(s);
  free(qf);
  free(acc_v);
  return ORACLE_OK;
}

int oracle_paged_attn_partial(const oracle_problem* p, const double* q, const uint8_t* k_cache,
                              const uint8_t* v_cache, const double* k_scale,
                              const double* v_scale, const int32_t* block_table,
                              const int32_t* seqlens_k, const int32_t* cu_seqlens_q,
                              const int32_t* key_begin, const int32_t* key_end, double* o,
                              double* lse) {
  if (check_problem(p, seqlens_k, cu_seqlens_q) != ORACLE_OK) return ORACLE_EINVAL;
  if (check_block_table(p, block_table, seqlens_k) != ORACLE_OK) return ORACLE_EINVAL;
  const int H = p->num_heads, D = p->head_size, G = p->num_heads / p->kv_num_heads;
  const double scale = softmax_scale_of(p);
  int maxL = 0;
  for (int b = 0; b < p->batch; ++b)
    if (seqlens_k[b] > maxL) maxL = seqlens_k[b];
  double* s = (double*)malloc(sizeof(double) * (maxL > 0 ? maxL : 1));
  if (!s) return ORACLE_EINVAL;
  for (int b = 0; b < p->batch; ++b) {
    const int Lb = seqlens_k[b];
    const int qb = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
    for (int i = 0; i < qb; ++i) {
      const int nk = visible_keys(p, Lb, qb, i);
      const int t0 = key_begin[b] > 0 ? key_begin[b] : 0;
      const int t1 = key_end[b] < nk ? key_end[b] : nk;
      const int64_t tok = cu_seqlens_q[b] + i;
      for (int h = 0; h < H; ++h) {
        const int kv = h / G;
        const double* qrow = q + (tok * H + h) * D;
        double* orow = o + (tok * H + h) * D;
        for (int d = 0; d < D; ++d) orow[d] = 0.0;
        if (t1 <= t0) {
          lse[tok * H + h] = -INFINITY;
          continue;
        }
        double smax = -INFINITY;
        for (int t = t0; t < t1; ++t) {
          const uint8_t* krow = cache_row(p, k_cache, block_table, b, t, kv);
          double acc = 0.0;
          for (int d = 0; d < D; ++d)
            acc += qrow[d] * (k_scale[kv * D + d] * oracle_decode(p->kv_dtype, krow, d));
          s[t] = scale * acc;
          if (s[t] > smax) smax = s[t];
        }
        double denom = 0.0;
        for (int t = t0; t < t1; ++t) {
          s[t] = exp(s[t] - smax);
          denom += s[t];
        }
        for (int t = t0; t < t1; ++t) {
          const uint8_t* vrow = cache_row(p, v_cache, block_table, b, t, kv);
          const double w = s[t] / denom;
          for (int d = 0; d < D; ++d)
            orow[d] += w * (v_scale[kv * D + d] * oracle_decode(p->kv_dtype, vrow, d));
        }
        lse[tok * H + h] = smax + log(denom);
      }
    }
  }
  free(s);
  return ORACLE_OK;
}

int oracle_lse_combine(int n_splits, int64_t rows, int head_size, const double* o_parts,
                       const double* lse_parts, double* out) {
  if (n_splits <= 0 || rows < 0 || head_size <= 0) return ORACLE_EINVAL;
  for (int64_t r = 0; r < rows; ++r) {
    /* lse = log sum_s exp(lse_s), evaluated around the largest term */
    double mx = -INFINITY;
    for (int sp = 0; sp < n_splits; ++sp)
      if (lse_parts[sp * rows + r] > mx) mx = lse_parts[sp * rows + r];
    double* orow = out + r * head_size;
    for (int d = 0; d < head_size; ++d) orow[d] = 0.0;
    if (mx == -INFINITY) continue; /* no split saw a key: cannot happen for a real row */
    double sum = 0.0;
    for (int sp = 0; sp < n_splits; ++sp) sum += exp(lse_parts[sp * rows + r] - mx);
    const double lse = mx + log(sum);
    for (int sp = 0; sp < n_splits; ++sp) {
      const double w = exp(lse_parts[sp * rows + r] - lse);
      if (w == 0.0) continue;
      for (int d = 0; d < head_size; ++d) orow[d] += w * o_parts[(sp * rows + r) * head_size + d];
    }
  }
  return ORACLE_OK;
}

int oracle_gather_decode(const oracle_problem* p, const uint8_t* cache,
                         const int32_t* block_table, const int32_t* seqlens_k, int b, int kv,
                         double* dst) {
  if (b < 0 || b >= p->batch || kv < 0 || kv >= p->kv_num_heads) return ORACLE_EINVAL;
  if (check_block_table(p, block_table, seqlens_k) != ORACLE_OK) return ORACLE_EINVAL;
  const int D = p->head_size;
  for (int t = 0; t < seqlens_k[b]; ++t) {
    const uint8_t* row = cache_row(p, cache, block_table, b, t, kv);
    for (int d = 0; d < D; ++d) dst[(int64_t)t * D + d] = oracle_decode(p->kv_dtype, row, d);
  }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------ writer */

/* Nearest e4m3fn value by brute force over the non-negative finite codes
 * (ascending), ties to the code with the even mantissa; beyond 448 the nearest
 * is 448 itself, which is the saturation. */
static int encode_e4m3(float q) {
  if (isnan(q)) return 0x7F;
  if (isinf(q)) return (signbit(q) ? 0x80 : 0) | 0x7E; /* saturation (no infinity code) */
  const double a = fabs((double)q);
  int best = 0;
  double best_d = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    const double d = fabs(decode_e4m3((uint8_t)c) - a);
    if (d < best_d || (d == best_d && (c & 1) == 0)) {
      best = c;
      best_d = d;
    }
  }
  return (signbit(q) ? 0x80 : 0) | best;
}

int oracle_quantise(int kv_dtype, float x, float s) {
  /* The symmetric code of x is the nearest code to x / s (value = scale x code),
   * with the quotient taken in IEEE single precision: one correctly rounded
   * division, no contraction. */
  const float q = x / s;
  if (kv_dtype == ORACLE_KV_FP8_E4M3) return encode_e4m3(q);
  if (isnan(q)) return 0;
  const int lo = kv_dtype == ORACLE_KV_INT4 ? -8 : -127;
  const int hi = kv_dtype == ORACLE_KV_INT4 ? 7 : 127;
  const float r = rintf(q); /* nearest, ties to even (default rounding mode) */
  if (r < (float)lo) return lo;
  if (r > (float)hi) return hi;
  return (int)r;
}

static void store_code(const oracle_problem* p, uint8_t* row, int d, int code) {
  if (p->kv_dtype == ORACLE_KV_INT4) {
    /* channel 2j low nibble, 2j+1 high nibble of byte j */
    const uint8_t nib = (uint8_t)(code & 0xF);
    if (d % 2 == 0)
      row[d / 2] = (uint8_t)((row[d / 2] & 0xF0) | nib);
    else
      row[d / 2] = (uint8_t)((row[d / 2] & 0x0F) | (nib << 4));
  } else {
    row[d] = (uint8_t)code;
  }
}

int oracle_append(const oracle_problem* p, const double* k_new, const double* v_new,
                  const float* k_scale, const float* v_scale, const int32_t* block_table,
                  const int32_t* seqlens_k, const int32_t* cu_seqlens_q, uint8_t* k_cache,
                  uint8_t* v_cache) {
  if (check_problem(p, seqlens_k, cu_seqlens_q) != ORACLE_OK) return ORACLE_EINVAL;
  if (check_block_table(p, block_table, seqlens_k) != ORACLE_OK) return ORACLE_EINVAL;
  const int Hk = p->kv_num_heads, D = p->head_size;
  for (int b = 0; b < p->batch; ++b) {
    const int q0 = cu_seqlens_q[b], qb = cu_seqlens_q[b + 1] - q0, Lb = seqlens_k[b];
    for (int i = 0; i < qb; ++i) {
      const int t = (Lb - qb) + i; /* absolute position of new token i */
      for (int kv = 0; kv < Hk; ++kv) {
        uint8_t* krow = (uint8_t*)cache_row(p, k_cache, block_table, b, t, kv);
        uint8_t* vrow = (uint8_t*)cache_row(p, v_cache, block_table, b, t, kv);
        const int64_t src = ((int64_t)(q0 + i) * Hk + kv) * D;
        for (int d = 0; d < D; ++d) {
          store_code(p, krow, d, oracle_quantise(p->kv_dtype, (float)k_new[src + d], k_scale[kv * D + d]));
          store_code(p, vrow, d, oracle_quantise(p->kv_dtype, (float)v_new[src + d], v_scale[kv * D + d]));
        }
      }
    }
  }
  return ORACLE_OK;
}
