/*
 * oracle.h -- plain FP64 CPU definition of paged grouped-query attention over
 * a low-precision (INT8 / packed INT4 / FP8-e4m3) KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library includes, links
 * or calls this code; only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load it.  It shares no source with the CUDA
 * path.  Every function is single-threaded, unblocked and unfused so that a
 * reader can check it against the definitions by eye.
 *
 * Sources (blog summaries of merged pull requests):
 *  [INT4-KV]  "ONNX Runtime: INT4 Paged KV Cache ... memory optimisation"
 *             (onnxruntime PR 32515), Code analysis 2 (cache shape and
 *             cache_head_size), Code analysis 3 (per-channel scale folded
 *             into Q, power-of-two normaliser).
 *  [INT8-TC]  "ONNX Runtime: Tensor-Core DynamicSparseAttention for INT8-KV
 *             cache" (onnxruntime PR 33707), "Why this is good" 2 (FP32
 *             accumulation checked against an FP64 reference).
 *  [MAXQ]     "[ONNX Runtime] PagedAttention FA path: exact max_query_len"
 *             (onnxruntime PR 28409), Code analysis 1 (ragged cum_q) and
 *             "Why this is good" (sequences with zero new tokens).
 *  [GEMV]     "Escaping the SGEMM trap: GQA GEMV decode kernel"
 *             (onnxruntime PR 29216), Code analysis 1 (tiling, online
 *             softmax, masking, flash-decoding structure), 2 (partials
 *             buffer), "Robust engineering: parity test".
 *  [FP8-PF]   "FlashInfer FP8 KV-Cache Prefill ... Repacking" (flashinfer
 *             PR 3485), introduction (1-byte FP8 KV cache).
 *
 * Parity status of each function is stated beside it ("pinned by ...").
 */
#ifndef PA_ORACLE_H
#define PA_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* KV element encodings. */
enum { ORACLE_KV_INT8 = 0, ORACLE_KV_INT4 = 1, ORACLE_KV_FP8_E4M3 = 2 };

/* Status codes: 0 ok, negative = contract violation (nothing written). */
enum { ORACLE_OK = 0, ORACLE_EINVAL = -1 };

/* Bytes per token per KV head in the cache: (head_size + 1) / 2 for packed
 * INT4, head_size otherwise ([INT4-KV] Code analysis 2). */
int oracle_cache_head_size(int kv_dtype, int head_size);

/* Exact value of channel d of one cache row (raw bytes, length chs).
 *  INT8: the signed byte.
 *  INT4: byte d/2; channel d is the low nibble when d is even, the high nibble
 *        when d is odd; 4-bit two's complement in [-8, 7].
 *  FP8 : OCP e4m3 ("fn"): bias 7, no infinities, S.1111.111 is NaN, max 448.
 * Pinned by: exhaustive INT4 pair round trip, all 256 e4m3 codes against the
 * format definition and torch's float8_e4m3fn decoder. */
double oracle_decode(int kv_dtype, const uint8_t* row, int d);

/* INT4 codec over `rows` rows of head_size channels.  pack: src int8 values in
 * [-8, 7] -> dst bytes [rows, (head_size+1)/2]; an odd head_size leaves the
 * last high nibble zero.  Returns ORACLE_EINVAL on an out-of-range value. */
int oracle_pack_int4(const int8_t* src, int64_t rows, int head_size, uint8_t* dst);
int oracle_unpack_int4(const uint8_t* src, int64_t rows, int head_size, int8_t* dst);

/* Problem description shared by the attention entry points. */
typedef struct {
  int batch, num_heads, kv_num_heads, head_size, block_size, num_blocks, max_blocks_per_seq;
  int kv_dtype;
  double softmax_scale;  /* 0 -> 1/sqrt(head_size) */
  int causal;            /* 1: new token i of sequence b sees keys t <= L_b - q_b + i */
} oracle_problem;

/* The definition, straight from the formula
 *    out = softmax(scale * Q * dequant(K)^T + causal mask) * dequant(V)
 * with dequant(x)[t, d] = scale[kv, d] * decode(x[block_table[b, t / bs],
 * t % bs, kv, :], d), kv = h / (num_heads / kv_num_heads).
 *  q      [T_q, H, D]  exact values of the fp16/bf16 queries
 *  k_cache, v_cache  [num_blocks, bs, Hk, chs] raw bytes
 *  k_scale, v_scale  [Hk, D] (exact values of the fp32 scales)
 *  block_table [B, max_blocks_per_seq], seqlens_k [B] (total keys, new ones
 *  included), cu_seqlens_q [B + 1] (packed new-token offsets).
 *  out [T_q, H, D]: rows of sequences with zero new tokens do not exist in
 *  the packed layout; nothing else is written.
 * Pinned by: Q = 0 mean, one-key, block permutation, contiguous brute force,
 * linearity in the scales, identical-group-heads, two-key closed form,
 * one-hot, split/combine equivalence (all in tests/test_oracle.py). */
int oracle_paged_attn(const oracle_problem* p, const double* q, const uint8_t* k_cache,
                      const uint8_t* v_cache, const double* k_scale, const double* v_scale,
                      const int32_t* block_table, const int32_t* seqlens_k,
                      const int32_t* cu_seqlens_q, double* out);

/* Same result computed the way the fused kernel reorganises it: the K scale is
 * folded into the query, q'[d] = q[d] * k_scale[kv, d] / 2^e with 2^e the
 * power of two of max_d |k_scale[kv, d]| (frexp exponent), and 2^e moved into
 * the logit multiplier ([INT4-KV] Code analysis 3); the V scale is applied once
 * to the weighted sum of raw decoded V values.  Exact algebra, so it must equal
 * oracle_paged_attn to FP64 rounding.  Pinned by: equality with the definition. */
int oracle_paged_attn_folded(const oracle_problem* p, const double* q, const uint8_t* k_cache,
                             const uint8_t* v_cache, const double* k_scale,
                             const double* v_scale, const int32_t* block_table,
                             const int32_t* seqlens_k, const int32_t* cu_seqlens_q,
                             double* out);

/* Partial attention of every new-token row over only the keys t in
 * [key_begin[b], key_end[b]) (further restricted by the causal/length limit):
 * o[row, d] = sum_t w_t v_hat[t, d] / sum_t w_t with w_t = exp(s_t - m) and
 * lse[row] = m + log(sum_t w_t) (natural log).  An empty key set gives
 * lse = -inf and o = 0.  This is the per-worker result of the flash-decoding
 * KV split ([GEMV] Code analysis 2, "partials buffer"). */
int oracle_paged_attn_partial(const oracle_problem* p, const double* q, const uint8_t* k_cache,
                              const uint8_t* v_cache, const double* k_scale,
                              const double* v_scale, const int32_t* block_table,
                              const int32_t* seqlens_k, const int32_t* cu_seqlens_q,
                              const int32_t* key_begin, const int32_t* key_end, double* o,
                              double* lse);

/* Log-sum-exp merge of n_splits partials [n_splits, rows, D] / [n_splits, rows]:
 * lse = log sum_s exp(lse_s); out = sum_s exp(lse_s - lse) o_s.  Splits with
 * lse_s = -inf carry weight 0.  Pinned by: split-vs-unsplit equality. */
int oracle_lse_combine(int n_splits, int64_t rows, int head_size, const double* o_parts,
                       const double* lse_parts, double* out);

/* Cache code of one new value x under per-channel scale s, for the
 * quantise-and-append writer that fills the cache the attention reads (INT4
 * paged-KV page, Code analysis 2: the cache holds per-channel symmetric codes,
 * value = scale x code).  The code is the nearest code to the quotient x / s,
 * the plain definition of a symmetric code, with the quotient taken in IEEE
 * single precision (one correctly rounded division):
 *   INT8: nearest integer to q (ties to even), clamped to [-127, 127];
 *   INT4: the same, clamped to [-8, 7] (the two's complement nibble);
 *   FP8 : the OCP e4m3fn value nearest to q (ties to the even mantissa),
 *         magnitudes past 448 saturated to 448; the sign of q is kept on 0.
 * A NaN quotient gives code 0 (integer caches) or 0x7F (FP8).  Readings (the
 * pages give the format, not the rounding): round to nearest even, symmetric
 * INT8 range, saturation, the quotient rounded once to fp32.  Returns the
 * signed code (INT8 / INT4) or the byte (FP8).  Pinned by: exact codes at
 * power-of-two scales, ties, saturation, the decode table round trip, torch's
 * e4m3fn cast, and codes next to a rounding boundary decided from the exact
 * rational quotient (where x times a rounded 1 / s lands on the other side). */
int oracle_quantise(int kv_dtype, float x, float s);

/* Quantise-and-append: the new K and V rows of every sequence ([T_q, Hk, D]
 * exact values, packed by cu_seqlens_q) are quantised with oracle_quantise
 * under k_scale / v_scale [Hk, D] and written at cache slot
 * block_table[b, t / bs] * bs + t % bs of absolute position t = L_b - q_b + i
 * for new token i (the cache layout of the INT4 paged-KV page, Code analysis
 * 2; INT4 channel 2j in the low nibble of byte j).  Every other cache byte is
 * left as it was.  Contract violations (lengths, block ids) write nothing and
 * return ORACLE_EINVAL.  Pinned by: placement into a sentinel cache, decode of
 * the written rows, untouched bytes. */
int oracle_append(const oracle_problem* p, const double* k_new, const double* v_new,
                  const float* k_scale, const float* v_scale, const int32_t* block_table,
                  const int32_t* seqlens_k, const int32_t* cu_seqlens_q, uint8_t* k_cache,
                  uint8_t* v_cache);

/* Keys of sequence b, dequantised and gathered into contiguous rows:
 * dst[t, d] = decode(cache[block_table[b, t / bs], t % bs, kv, :], d) for
 * t < seqlens_k[b], WITHOUT the per-channel scale (exact small values).
 * Pinned by: block permutation and the contiguous brute force. */
int oracle_gather_decode(const oracle_problem* p, const uint8_t* cache,
                         const int32_t* block_table, const int32_t* seqlens_k, int b, int kv,
                         double* dst);

#ifdef __cplusplus
}
#endif
#endif /* PA_ORACLE_H */
