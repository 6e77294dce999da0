/*
 * paged_attn.h -- C ABI of the B200 (sm_100a) paged quantised-KV attention library
 * (libpagedattn.so).
 *
 * Operation.  Grouped-query attention of the new tokens of a ragged batch over a
 * paged low-precision KV cache:
 *
 *     out = softmax(scale * Q * dequant(K)^T + causal mask) * dequant(V)
 *
 * Sources (blog summaries of merged pull requests; cited by title and section):
 *  - "ONNX Runtime: INT4 Paged KV Cache ... memory optimisation" (onnxruntime
 *    PR 32515), Code analysis 2: cache shape (num_blocks, block_size,
 *    kv_num_heads, cache_head_size) with cache_head_size = (head_size + 1) / 2 for
 *    packed INT4 and head_size otherwise; Code analysis 3: the per-channel K
 *    scale is folded into Q, normalised by the power of two of max|k_scale| so
 *    fp16 cannot overflow.
 *  - "ONNX Runtime: Tensor-Core DynamicSparseAttention for INT8-KV cache"
 *    (onnxruntime PR 33707), Code analysis 1: INT8 kept raw until it is
 *    converted to FP16 in registers right before the tensor-core MMA, FP32
 *    accumulation.
 *  - "[ONNX Runtime] PagedAttention FA path: exact max_query_len" (onnxruntime
 *    PR 28409), Code analysis 1-2: the launch is sized by the exact host-side
 *    max over b of cu_seqlens_q[b+1] - cu_seqlens_q[b]; sequences with zero new
 *    tokens are legal.
 *  - "Escaping the SGEMM trap: GQA GEMV decode kernel" (onnxruntime PR 29216),
 *    Code analysis 2: flash decoding splits one sequence's keys across workers
 *    when batch x heads underfills the machine, with a partials buffer.
 *  - "FlashInfer FP8 KV-Cache Prefill ... Repacking" (flashinfer PR 3485):
 *    1-byte FP8 KV cache (read here as OCP e4m3fn).
 *
 * Besides the attention call the ABI has the cache writer that fills the cache
 * (paged_kv_append: new fp16/bf16 K/V rows -> per-channel codes at their slots)
 * and the log-sum-exp merge of results over disjoint key sets
 * (paged_attn_merge, with the forward call's optional per-row lse_out) for a
 * sequence whose keys are spread over several GPUs.
 *
 * Readings where the pages are silent (all of them are properties of this ABI):
 *  - seqlens_k[b] counts every key of sequence b, the new tokens included; the
 *    past length is seqlens_k[b] - q_b (q_b = new tokens of b).
 *  - Causal mask is bottom-right aligned: new token i of b sees keys
 *    t <= seqlens_k[b] - q_b + i.  For decode (q_b = 1) that is every key.
 *  - Query head h uses KV head h / (num_heads / kv_num_heads).
 *  - INT4: channel 2j is the low nibble of byte j, channel 2j+1 the high nibble,
 *    4-bit two's complement in [-8, 7].
 *  - Dequantisation is symmetric: value = scale[kv, d] * code, scales fp32
 *    [kv_num_heads, head_size], shared by every token and block.
 *
 * Memory layouts (all row-major, all device memory unless the name says _host):
 *  q, out        [total_q, num_heads, head_size] fp16 or bf16, tokens packed by
 *                cu_seqlens_q (sequence b owns rows cu[b] .. cu[b+1]-1).
 *  k_cache,
 *  v_cache       [num_blocks, block_size, kv_num_heads, cache_head_size] bytes.
 *                Base address 16-byte aligned.
 *  k_scale,
 *  v_scale       [kv_num_heads, head_size] fp32.
 *  block_table   [batch, max_blocks_per_seq] int32; entry (b, l) is the physical
 *                block holding keys l*block_size .. l*block_size+block_size-1.
 *  seqlens_k     [batch] int32.
 *  cu_seqlens_q  [batch + 1] int32, cu[0] = 0, non-decreasing.
 *
 * Ownership and state.  The caller owns every buffer, the workspace included.
 * The library allocates no memory and keeps no state between calls; every call
 * is asynchronous on the given stream (a cudaStream_t passed as void*; NULL is
 * the legacy default stream).  No exception crosses the ABI: each entry point
 * returns a pa_status, and paged_attn_last_error() gives a message for the last
 * failing call on the calling thread.
 *
 * Errors.  Argument and contract violations are detected on the host before
 * any launch and return PA_ERR_INVALID_ARG / PA_ERR_UNSUPPORTED /
 * PA_ERR_WORKSPACE.  A launch failure returns PA_ERR_CUDA.  Conditions that
 * only the device can see (a block-table entry outside [0, num_blocks), a
 * non-finite K or V scale, device lengths that contradict the plan, a pipeline
 * wait that timed out) never fault the GPU: the kernel reads zeros instead, finishes,
 * and ORs a bit into the sticky error word at the start of the workspace, which
 * paged_attn_read_device_error() returns.
 */
#ifndef PAGED_ATTN_H
#define PAGED_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = -1,     /* bad pointer, size, or contract violation */
  PA_ERR_UNSUPPORTED = -2,     /* valid request outside the compiled set */
  PA_ERR_WORKSPACE = -3,       /* workspace missing or smaller than planned */
  PA_ERR_BAD_BLOCK_TABLE = -4, /* device error word: block id out of range */
  PA_ERR_CUDA = -5,            /* CUDA runtime / launch error */
  PA_ERR_DEVICE = -6           /* device error word: other device-side condition */
} pa_status;

typedef enum { PA_KV_INT8 = 0, PA_KV_INT4 = 1, PA_KV_FP8_E4M3 = 2 } pa_kv_dtype;
/* Element types of q, out and the merge operands.  PA_F32 is an output type only
 * (out of paged_attn_forward, the parts of paged_attn_merge): the unrounded rows
 * of a partial result that another call merges. */
typedef enum { PA_F16 = 0, PA_BF16 = 1, PA_F32 = 2 } pa_dtype;

/* Bits of the device error word (see paged_attn_read_device_error). */
#define PA_DEVERR_BAD_BLOCK 0x1u   /* block_table entry outside [0, num_blocks) */
#define PA_DEVERR_TIMEOUT 0x2u     /* an mbarrier wait exceeded its time bound */
#define PA_DEVERR_BAD_SCALE 0x4u   /* a K or V scale of a KV head is not finite */
#define PA_DEVERR_BAD_LENGTH 0x8u  /* device seqlens/cu_seqlens contradict the plan */

typedef struct {
  /* ---- problem description: filled by the caller ---- */
  int batch;              /* B >= 0 */
  int num_heads;          /* H, query heads */
  int kv_num_heads;       /* Hk, H % Hk == 0 */
  int head_size;          /* D: 64 or 128 */
  int block_size;         /* tokens per cache block: 16 or 32 */
  int num_blocks;         /* physical blocks in each cache pool */
  int max_blocks_per_seq; /* columns of block_table */
  int kv_dtype;           /* pa_kv_dtype */
  int q_dtype;            /* pa_dtype of q: PA_F16 or PA_BF16 */
  int out_dtype;          /* pa_dtype of out: PA_F16, PA_BF16 or PA_F32 (out then
                             16-byte aligned) */
  float softmax_scale;    /* 0 -> 1/sqrt(head_size) */
  int causal;             /* 1: bottom-right causal mask for new tokens; 0: none */
  int num_sms;            /* 0 -> SM count of the current device (148 if none) */
  int split_blocks;       /* 0: planner decides; > 0: use this split target T (KV
                             blocks per split); < 0: never split */
  /* ---- filled by paged_attn_plan ---- */
  int total_q;            /* cu_seqlens_q[batch] */
  int max_query_len;      /* exact max_b (cu[b+1] - cu[b]) */
  int max_seqlen_k;       /* max_b seqlens_k[b] */
  int rows_per_cta;       /* query rows (tokens x group heads) per work item: 4, 8
                             or 16 (4: at most 4 rows per sequence and KV head),
                             or 64: the tensor-core prefill kernel, chosen when a
                             unit has more than 16 rows over an INT8 cache with
                             head_size 128 and batch <= 1024 */
  int num_row_groups;     /* ceil(max_query_len * H/Hk / rows_per_cta) */
  int num_splits;         /* most KV splits of any sequence (1 = no split); the
                             workspace holds this many partials per row */
  int blocks_per_split;   /* split target T in KV blocks: a sequence with n blocks
                             is cut into min(num_splits, ceil(n / T)) equal splits */
  int num_work_items;     /* work items (sequence, KV heads, row group, split): four
                             KV heads per item on the 4/8/16-row kernel, one on
                             the prefill kernel */
  size_t workspace_bytes; /* bytes the forward call needs (>= 256) */
  /* ---- supplied by the caller before paged_attn_forward ---- */
  void* workspace;        /* device memory, 256-byte aligned, >= workspace_bytes,
                             zeroed once with paged_attn_workspace_init; holds the
                             error word, the work counters (they return to zero at
                             the end of every call) and the split partials.
                             Calls that share a workspace must not overlap on the
                             GPU. */
  void* profile_events;   /* optional profiling hook: NULL, or a pointer to two
                             cudaEvent_t that paged_attn_forward records on the
                             stream right before and right after the fused
                             attention kernel launch */
  int stall_consumers;    /* diagnostic, 0 normally.  1: the decode kernel's
                             consumer warps wait on a barrier that nothing
                             signals, so that the bounded-wait path runs: the
                             call takes about two seconds (the waits' bound),
                             sets PA_DEVERR_TIMEOUT, leaves the output rows
                             undefined and the GPU context usable; re-initialise
                             the workspace before the next call. */
  float* lse_out;         /* optional: NULL, or device [total_q, num_heads] fp32
                             that receives each row's log-sum-exp of its scaled
                             logits, log sum_t exp(s_t) (natural log; -inf when the
                             row sees no key), so that results over disjoint key
                             sets merge exactly (paged_attn_merge; the GQA GEMV
                             decode page, Code analysis 2) */
} paged_attn_params;

/* Host-side planner.  Validates the problem, computes the exact max_query_len
 * and max_seqlen_k from HOST copies of cu_seqlens_q [batch+1] and seqlens_k
 * [batch] (the exact-max_query_len page, Code analysis 1), chooses the KV split
 * (flash decoding after the GQA GEMV decode page's rule: the split target that
 * makes the work items fill the device's resident CTA slots in the least
 * estimated time; no split when the units alone do), and
 * reports the workspace size.  Launches nothing; needs no GPU.  Contract checks:
 * cu[0] == 0, 0 <= q_b <= seqlens_k[b] <= max_blocks_per_seq * block_size. */
pa_status paged_attn_plan(const int32_t* cu_seqlens_q_host, const int32_t* seqlens_k_host,
                          paged_attn_params* params, size_t* workspace_bytes_needed);

/* Attention forward (see the header comment for layouts).  params must come from
 * paged_attn_plan with the same lengths the device arrays hold.  total_q == 0
 * returns PA_OK without a launch.  Rows of sequences with q_b == 0 do not exist
 * in q/out; no other byte of out is written.  One kernel launch per call, plus,
 * when params->num_splits > 1, a log-sum-exp combine of the split partials
 * launched as the forward kernel's programmatic dependent (it overlaps the
 * forward kernel's tail and waits for its completion).  q, k_scale
 * and v_scale must be 16-byte aligned, the caches 16-byte aligned, out 4-byte
 * aligned.  After a device error the workspace should be re-initialised.
 * Extreme scales (the INT4 paged-KV page's lesson on FLT_MAX scales): K scales
 * and queries of any finite magnitude, up to FLT_MAX, give finite outputs that
 * follow the definition (when the logits leave fp32 range the softmax is the
 * hard maximum it tends to); a NaN or infinite K or V scale sets
 * PA_DEVERR_BAD_SCALE and the output rows are then undefined.  Outputs whose
 * true value exceeds the output type's range round to +-infinity. */
pa_status paged_attn_forward(const void* q, const void* k_cache, const void* v_cache,
                             const float* k_scale, const float* v_scale,
                             const int32_t* block_table, const int32_t* seqlens_k,
                             const int32_t* cu_seqlens_q, void* out,
                             const paged_attn_params* params, void* stream);

/* Size of the library-owned scratch used by paged_attn_forward_noalloc: 16 MiB,
 * held by every GPU that loads the library until the process exits. */
#define PA_NOALLOC_MAX_WORKSPACE_BYTES (16u << 20)

/* paged_attn_forward for callers that cannot allocate device memory.  (The
 * pages have no counterpart: this entry point exists for the caller's memory
 * model, not for the method.)
 *
 * Who needs it: code that must not call cudaMalloc or any allocator where it
 * runs attention -- an operator inside a host framework that owns every device
 * buffer, a fixed memory plan replayed step after step, a real-time loop whose
 * memory is frozen at start-up.  Such callers hold q, the caches, the scales,
 * the block table, the lengths and out, but have no workspace to give.
 *
 * What it does: the same computation and kernel launch as paged_attn_forward
 * (same arguments, layouts and results), with the workspace taken from a
 * library-owned device array of PA_NOALLOC_MAX_WORKSPACE_BYTES instead of
 * params->workspace (which is ignored).  It allocates and frees nothing.
 *  - params must come from paged_attn_plan; if its workspace_bytes exceeds
 *    PA_NOALLOC_MAX_WORKSPACE_BYTES the call returns PA_ERR_WORKSPACE before any
 *    device work (plan again with a larger split_blocks, i.e. fewer splits, or
 *    use paged_attn_forward with your own workspace).
 *  - Every call looks up the array's device address on the current device
 *    (cudaGetSymbolAddress, a host-side query that allocates nothing).  The
 *    first lookup on a device loads the library's device code there: make the
 *    first call on a device before any stream capture on it.
 *  - Every call clears the array's error word and counters on `stream`
 *    (cudaMemsetAsync) before the launch; the array keeps the rest of the last
 *    call's contents.  paged_attn_read_device_error(NULL, ...) reads (and
 *    optionally clears) the array's error word on the current device, so the
 *    device-side conditions of the last call are visible until the next call
 *    clears them.
 *  - All calls in the process share the one array per device: calls whose
 *    executions overlap on the GPU (different streams without ordering between
 *    them) race on it and give wrong results.  Order them on one stream. */
pa_status paged_attn_forward_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                     const float* k_scale, const float* v_scale,
                                     const int32_t* block_table, const int32_t* seqlens_k,
                                     const int32_t* cu_seqlens_q, void* out,
                                     const paged_attn_params* params, void* stream);

/* Zero a workspace (the sticky error word and all scratch).  Call once after
 * allocating it; asynchronous on stream. */
pa_status paged_attn_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Synchronise `stream`, read the device error word from `workspace` into *bits
 * (PA_DEVERR_* flags), and zero it when `clear` is non-zero.  workspace NULL
 * reads the word of paged_attn_forward_noalloc's library-owned scratch on the
 * current device.  Returns PA_OK when no bit is set, PA_ERR_BAD_BLOCK_TABLE
 * when PA_DEVERR_BAD_BLOCK is set, and PA_ERR_DEVICE for any other bit.  After
 * PA_DEVERR_BAD_LENGTH (device lengths that contradict the plan) the rows of the
 * offending sequences are undefined: out may hold values left from an earlier
 * call sharing the workspace. */
pa_status paged_attn_read_device_error(void* workspace, int clear, uint32_t* bits, void* stream);

/* INT4 codec (INT4 paged-KV page, Code analysis 2).  pack: int8 values in
 * [-8, 7], [rows, head_size] -> bytes [rows, head_size/2] with channel 2j in the
 * low nibble.  unpack: the inverse.  head_size must be even.  A value outside
 * [-8, 7] is packed from its low 4 bits (the kernel does not check). */
pa_status paged_kv_pack_int4(const int8_t* src, uint8_t* dst, int64_t rows, int head_size,
                             void* stream);
pa_status paged_kv_unpack_int4(const uint8_t* src, int8_t* dst, int64_t rows, int head_size,
                               void* stream);

/* Log-sum-exp merge of attention results over disjoint key sets (the flash-
 * decoding combine of the GQA GEMV decode page, Code analysis 2, across calls:
 * context parallelism, one key range per GPU).  parts: [n_parts, rows,
 * head_size] of parts_dtype (PA_F16, PA_BF16 or PA_F32), each part normalised
 * over its own keys; lse_parts: [n_parts, rows] fp32, natural log, -inf for a
 * part with no key (as paged_attn_forward's lse_out gives them).  out[r] =
 * sum_p exp(lse_p[r] - lse[r]) parts[p, r] with lse[r] = log sum_p
 * exp(lse_p[r]), accumulated in fp32 and rounded to out_dtype (PA_F16 or
 * PA_BF16); a row with no key in any part gets zeros.  lse_out (optional,
 * [rows]) receives lse.  1 <= n_parts <= 64; head_size 64 or 128; device
 * pointers, parts/out 8-byte aligned (16-byte for PA_F32 parts); async on
 * `stream`. */
pa_status paged_attn_merge(const void* parts, int parts_dtype, const float* lse_parts,
                           int n_parts, int64_t rows, int head_size, void* out, int out_dtype,
                           float* lse_out, void* stream);

/* Quantise-and-append: the cache write that precedes the attention call (the
 * INT4 paged-KV page, Code analysis 2-3: per-channel symmetric codes,
 * value = scale x code, in the [num_blocks, block_size, Hk, chs] cache).
 *
 * For every sequence b and new token i < q_b (q_b from cu_seqlens_q), at
 * absolute position t = seqlens_k[b] - q_b + i, the K and V rows of that token
 * (k_new / v_new, [total_q, Hk, head_size] in params->q_dtype, packed by
 * cu_seqlens_q like q) are stored at cache slot block_table[b, t / block_size]
 * * block_size + t % block_size, head kv.  Channel d's code is decided in IEEE
 * single precision from q = x / scale[kv, d] (correctly rounded division):
 *   INT8: nearest integer (ties to even) clamped to [-127, 127];
 *   INT4: the same clamped to [-8, 7], channel 2j in the low nibble of byte j;
 *   FP8 : round-to-nearest-even e4m3fn, saturating at +-448.
 * A NaN quotient stores 0 (integer caches) or 0x7F (FP8).  No other cache byte
 * is written.
 *
 * params: the plan of the same call (paged_attn_plan sets total_q); batch,
 * kv_num_heads, head_size, block_size, num_blocks, max_blocks_per_seq,
 * kv_dtype and q_dtype are read, and params->workspace (device, 256-byte
 * aligned, >= 256 bytes) holds the device error word of byte 0 as for
 * paged_attn_forward.  All array pointers are device pointers; k_new, v_new,
 * the scales and the caches must be 16-byte aligned.  The caller owns every
 * buffer.  A row whose sequence lengths are invalid or whose block id lies
 * outside [0, num_blocks) is not written and sets PA_DEVERR_BAD_LENGTH /
 * PA_DEVERR_BAD_BLOCK in the error word (read with
 * paged_attn_read_device_error).  Host-checked violations return an error
 * status with nothing launched; total_q == 0 returns PA_OK.  Asynchronous on
 * `stream`. */
pa_status paged_kv_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                          const float* k_scale, const float* v_scale, const int32_t* block_table,
                          const int32_t* seqlens_k, const int32_t* cu_seqlens_q,
                          const paged_attn_params* params, void* stream);

/* Test hook: gather the keys (or values) of sequence b, KV head kv through the
 * block table, decode them with the attention kernel's conversion routines and
 * store the exact unscaled codes as fp16 (dst_dtype PA_F16) or bf16 (PA_BF16),
 * contiguous [seqlens_k[b], head_size].  `len_b` is the host value of
 * seqlens_k[b].  Every code of all three formats is exact in both types. */
pa_status paged_kv_gather_decode(const void* cache, const int32_t* block_table,
                                 const paged_attn_params* params, int b, int kv, int len_b,
                                 int dst_dtype, void* dst, void* stream);

/* Measurement helper: stream `bytes` (multiple of 16, 16-byte aligned) from
 * `src` with 16-byte loads on every SM and write one 16-byte checksum per block
 * to `sink` (>= 16 * 148 * 8 bytes).  The read-only HBM ceiling that the
 * attention kernel is compared against. */
pa_status paged_attn_stream_read(const void* src, size_t bytes, void* sink, void* stream);

/* Message for the last non-PA_OK status returned on this thread ("" if none). */
const char* paged_attn_last_error(void);

/* Library version string. */
const char* paged_attn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PAGED_ATTN_H */
