// pa_internal.h -- declarations shared by the host API and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "paged_attn.h"

namespace pa {

// Everything the fused forward kernel needs besides the two tensor maps.
struct FwdArgs {
  const void* q;
  void* out;
  const float* k_scale;
  const float* v_scale;
  const int32_t* block_table;
  const int32_t* seqlens_k;
  const int32_t* cu_seqlens_q;
  __half* o_part;       // [max_splits, total_q * H, D] fp16, code units (split mode only)
  float* lse_part;      // [max_splits, total_q * H] (log2 domain)
  int32_t* row_ns;      // [total_q * H] splits with keys of each row's unit (split mode only)
  float* lse_out;       // optional [total_q * H] natural-log log-sum-exp of each row
  uint32_t* frag;       // [batch * Hk * num_row_groups] precomputed query fragment units
  uint32_t* work;       // [2]: next work item, CTAs finished (both rewound by the last CTA)
  uint32_t* err;        // sticky device error word
  int batch, H, Hk, G, maxb, num_blocks, total_q;
  int q_bf16, out_bf16, out_f32, causal;  // out_f32: fp32 rows (for a later merge)
  int rows_cta;         // query rows per (KV head, row group): 4, 8 or 16
  int num_row_groups;   // largest number of row groups of a (sequence, KV head)
  int max_splits;       // partial slots: no sequence is split into more items
  int split_target;     // KV blocks per split target T: n blocks -> min(max_splits, ceil(n / T))
                        // equal splits of ceil(n / splits) blocks
  int num_items;        // work items of the plan (grid = min(num_items, resident CTAs))
  int num_sms;          // SMs of the device
  float sm_scale_log2;  // softmax_scale * log2(e)
  int stall_consumers;  // diagnostic: consumer warps wait on a barrier nothing signals
};

// KV heads of one work item: the fused kernel streams their rows of a block with
// one TMA box and gives each to one consumer warp.
constexpr int kHeadsPerItem = 4;

// Split geometry of a sequence with nblk KV blocks for split target T: the
// number of non-empty splits and the blocks per split.  Shared by the planner
// and the kernel so that both count the same items.
__host__ __device__ inline void split_geometry(int nblk, int T, int max_splits, int* nsplit,
                                               int* bps) {
  int s = (nblk + T - 1) / T;
  if (s < 1) s = 1;
  if (s > max_splits) s = max_splits;
  const int per = nblk > 0 ? (nblk + s - 1) / s : 1;
  *bps = per;
  *nsplit = nblk > 0 ? (nblk + per - 1) / per : 1;
}

// Workspace layout: [0, 256) header: error word at byte 0, work counters at
// byte 64; then the precomputed query fragments; then the split partial outputs
// and their log-sum-exps (256-byte aligned each).
constexpr size_t kWsHeaderBytes = 256;
constexpr size_t kWsWorkOffset = 64;

// Arguments of the quantise-and-append writer (pa_append.cu).
struct AppendArgs {
  const void* k_new;  // [total_q, Hk, D] fp16 / bf16
  const void* v_new;
  void* k_cache;      // [num_blocks, block_size, Hk, chs]
  void* v_cache;
  const float* k_scale;  // [Hk, D]
  const float* v_scale;
  const int32_t* block_table;
  const int32_t* seqlens_k;
  const int32_t* cu_seqlens_q;
  uint32_t* err;      // device error word (workspace byte 0)
  int batch, Hk, maxb, num_blocks, block_size, total_q;
  bool in_bf16;
};
cudaError_t launch_append(int kv_dtype, int head_size, const AppendArgs& a, cudaStream_t stream);
// Log-sum-exp merge of results over disjoint key sets (pa_append.cu).
cudaError_t launch_merge(const void* parts, int parts_dtype, const float* lse_parts, int n_parts,
                         long long rows, int head_size, bool out_bf16, void* out, float* lse_out,
                         cudaStream_t stream);

// Launcher (pa_attention.cu).  rows_per_cta is 4 (decode rows packed with their
// fp16 residuals), 8 or 16.
cudaError_t launch_forward(int kv_dtype, int head_size, int block_size, int rows_per_cta,
                           const CUtensorMap& kmap, const CUtensorMap& vmap, const FwdArgs& a,
                           cudaStream_t stream);
// Log-sum-exp merge of the split partials (one warp per row of a split unit),
// launched right after the forward kernel as its programmatic dependent.
cudaError_t launch_combine(int head_size, int block_size, const FwdArgs& a, cudaStream_t stream);
// Tensor-core prefill kernel (pa_prefill.cu): work items of up to 64 query rows
// of one KV head.  Supported for INT8 caches, head_size 128, block_size 16 or
// 32, batch <= 1024.
bool prefill_supported(int kv_dtype, int head_size, int block_size, int batch);
int prefill_rows_per_item();
// 32-bit words of one (sequence, KV head, row group) unit of query digits in
// the workspace (written by the prefill kernel's pre-pass).
int prefill_unit_words();
cudaError_t launch_prefill(int block_size, const CUtensorMap& kmap, const CUtensorMap& vmap,
                           const FwdArgs& a, cudaStream_t stream);
// Dynamic shared memory of one forward CTA (-1 for an unsupported combination).
int forward_smem_bytes(int kv_dtype, int head_size, int block_size, int rows_per_cta);
// 32-bit words of one precomputed query-fragment unit (sequence, KV head, row group).
int fragment_unit_words(int kv_dtype, int head_size, int rows_per_cta);
// Forward CTAs resident per SM, from the launch bounds and shared memory.
int forward_ctas_per_sm(int kv_dtype, int head_size, int block_size, int rows_per_cta);

// Device address, on the current device, of the library-owned scratch that
// paged_attn_forward_noalloc uses as its workspace (pa_noalloc.cu).
pa_status noalloc_scratch_address(void** out);

// Sets the thread's message for paged_attn_last_error() and returns st
// (pa_api.cu; used by entry points defined in other files).
pa_status set_last_error(pa_status st, const char* msg);

// Codec and measurement kernels (pa_codec.cu).
cudaError_t launch_pack_int4(const int8_t* src, uint8_t* dst, int64_t rows, int head_size,
                             cudaStream_t s);
cudaError_t launch_unpack_int4(const uint8_t* src, int8_t* dst, int64_t rows, int head_size,
                               cudaStream_t s);
cudaError_t launch_gather_decode(const uint8_t* cache, const int32_t* block_table, int kv_dtype,
                                 int head_size, int block_size, int kv_num_heads, int maxb,
                                 int num_blocks, int b, int kv, int len_b, int dst_bf16,
                                 void* dst, cudaStream_t s);
cudaError_t launch_stream_read(const void* src, size_t bytes, void* sink, cudaStream_t s);

}  // namespace pa
