// pa_api.cu -- host side of libpagedattn.so: argument checks, the planner,
// tensor-map encoding and launches.  Every entry point is extern "C", returns a
// pa_status and never throws.
//
// Planner sources: the exact host-side max_query_len replacing the heuristic
// token_count - batch_size + 1, which goes wrong (and negative) when sequences
// carry zero new tokens (exact max_query_len page, onnxruntime PR 28409, Code
// analysis 1 and "Why this is good"); explicit checks on values that cross a
// file boundary instead of asserts (same page, "Lessons" 1 and reviewer
// feedback); flash decoding chosen when batch x heads underfills the workers
// and there is more than one KV chunk (GQA GEMV decode page, onnxruntime PR
// 29216, Code analysis 2).
#include <cudaTypedefs.h>

#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "pa_internal.h"

namespace {

thread_local char g_last_error[512] = "";

pa_status fail(pa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

pa_status ok() {
  g_last_error[0] = '\0';
  return PA_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr size_t kHeaderBytes = pa::kWsHeaderBytes;  // error word + reserved
constexpr int kMaxSplits = 128;        // merge weights of one row group fit in shared memory
constexpr double kItemCostBytes = 16384.0;  // fixed cost of one work item, in KV bytes

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace layout shared by the planner and the forward call.
struct WsLayout {
  size_t frag, o_part, lse_part, row_ns, total;
};

WsLayout ws_layout(const paged_attn_params* p) {
  WsLayout w;
  size_t off = kHeaderBytes;
  w.frag = off;
  const size_t units = static_cast<size_t>(p->batch) * p->kv_num_heads * p->num_row_groups;
  const int uw = pa::fragment_unit_words(p->kv_dtype, p->head_size, p->rows_per_cta);
  off = align256(off + units * static_cast<size_t>(uw > 0 ? uw : 0) * 4);
  if (p->num_splits > 1) {
    w.o_part = off;
    const size_t rows = static_cast<size_t>(p->total_q) * p->num_heads;
    off = align256(off + rows * p->num_splits * p->head_size * 2);  // fp16 partials
    w.lse_part = off;
    off = align256(off + rows * p->num_splits * sizeof(float));
    w.row_ns = off;  // each row's split count
    off = align256(off + rows * sizeof(int32_t));
  } else {
    w.o_part = w.lse_part = w.row_ns = 0;
  }
  w.total = off;
  return w;
}

int cache_row_bytes(int kv_dtype, int head_size) {
  return kv_dtype == PA_KV_INT4 ? (head_size + 1) / 2 : head_size;
}

pa_status check_problem(const paged_attn_params* p) {
  if (p == nullptr) return fail(PA_ERR_INVALID_ARG, "params is NULL");
  if (p->batch < 0) return fail(PA_ERR_INVALID_ARG, "batch %d < 0", p->batch);
  if (p->num_heads <= 0 || p->kv_num_heads <= 0)
    return fail(PA_ERR_INVALID_ARG, "num_heads %d / kv_num_heads %d must be > 0", p->num_heads,
                p->kv_num_heads);
  if (p->num_heads % p->kv_num_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "num_heads %d is not a multiple of kv_num_heads %d",
                p->num_heads, p->kv_num_heads);
  if (p->kv_dtype < PA_KV_INT8 || p->kv_dtype > PA_KV_FP8_E4M3)
    return fail(PA_ERR_INVALID_ARG, "unknown kv_dtype %d", p->kv_dtype);
  if (p->q_dtype != PA_F16 && p->q_dtype != PA_BF16)
    return fail(PA_ERR_INVALID_ARG, "q_dtype must be PA_F16 or PA_BF16");
  if (p->out_dtype != PA_F16 && p->out_dtype != PA_BF16 && p->out_dtype != PA_F32)
    return fail(PA_ERR_INVALID_ARG, "out_dtype must be PA_F16, PA_BF16 or PA_F32");
  if (p->head_size <= 0 || p->block_size <= 0 || p->num_blocks < 0 || p->max_blocks_per_seq < 0)
    return fail(PA_ERR_INVALID_ARG, "head_size, block_size must be > 0 and counts >= 0");
  if (p->head_size != 64 && p->head_size != 128)
    return fail(PA_ERR_UNSUPPORTED, "head_size %d not in {64, 128}", p->head_size);
  if (p->block_size != 16 && p->block_size != 32)
    return fail(PA_ERR_UNSUPPORTED, "block_size %d not in {16, 32}", p->block_size);
  if (!(p->softmax_scale >= 0.f) || isinf(p->softmax_scale))
    return fail(PA_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0 (0 = default)");
  if (static_cast<int64_t>(p->num_blocks) * p->block_size >= (int64_t(1) << 31))
    return fail(PA_ERR_UNSUPPORTED, "num_blocks * block_size must stay below 2^31 tokens");
  if (p->causal != 0 && p->causal != 1) return fail(PA_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (p->stall_consumers != 0 && p->stall_consumers != 1)
    return fail(PA_ERR_INVALID_ARG, "stall_consumers must be 0 or 1");
  return PA_OK;
}

int current_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

pa_status get_encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::call_once(g_encode_once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  });
  if (g_encode == nullptr)
    return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  *fn = g_encode;
  return PA_OK;
}

// 3-D view of one cache pool: (cache_head_size bytes, num_blocks * block_size
// tokens, kv_num_heads); the box is 16 tokens of `box_heads` heads (4 for the
// decode kernel, 1 for the prefill kernel), heads outermost in shared memory so
// that each head's rows are contiguous there.
pa_status encode_cache_map(const void* cache, const paged_attn_params* p, int box_heads,
                           CUtensorMap* map) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  pa_status st = get_encoder(&enc);
  if (st != PA_OK) return st;
  const int chs = cache_row_bytes(p->kv_dtype, p->head_size);
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(chs),
                        static_cast<cuuint64_t>(p->num_blocks) * p->block_size,
                        static_cast<cuuint64_t>(p->kv_num_heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(chs) * p->kv_num_heads,
                           static_cast<cuuint64_t>(chs)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(chs), 16u, static_cast<cuuint32_t>(box_heads)};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUtensorMapSwizzle swz = chs == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : chs == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                             : CU_TENSOR_MAP_SWIZZLE_32B;
  const CUtensorMapL2promotion promo =
      chs >= 128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                 : (chs >= 64 ? CU_TENSOR_MAP_L2_PROMOTION_L2_64B : CU_TENSOR_MAP_L2_PROMOTION_NONE);
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(cache), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, promo,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return PA_OK;
}

pa_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return PA_OK;
  return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace

pa_status pa::set_last_error(pa_status st, const char* msg) {
  snprintf(g_last_error, sizeof(g_last_error), "%s", msg);
  return st;
}

extern "C" {

const char* paged_attn_last_error(void) { return g_last_error; }

const char* paged_attn_version(void) { return "paged_quantized_kv_attention_b200 0.1 (sm_100a)"; }

pa_status paged_attn_plan(const int32_t* cu_seqlens_q_host, const int32_t* seqlens_k_host,
                          paged_attn_params* p, size_t* workspace_bytes_needed) {
  pa_status st = check_problem(p);
  if (st != PA_OK) return st;
  if (p->batch > 0 && (cu_seqlens_q_host == nullptr || seqlens_k_host == nullptr))
    return fail(PA_ERR_INVALID_ARG, "cu_seqlens_q_host / seqlens_k_host is NULL");
  const int B = p->batch, G = p->num_heads / p->kv_num_heads, bs = p->block_size;
  if (B > 0 && cu_seqlens_q_host[0] != 0)
    return fail(PA_ERR_INVALID_ARG, "cu_seqlens_q[0] = %d, expected 0", cu_seqlens_q_host[0]);
  int max_q = 0, max_k = 0;
  int64_t total_blocks = 0;
  for (int b = 0; b < B; ++b) {
    const int qb = cu_seqlens_q_host[b + 1] - cu_seqlens_q_host[b];
    const int Lb = seqlens_k_host[b];
    if (qb < 0) return fail(PA_ERR_INVALID_ARG, "cu_seqlens_q decreases at b=%d", b);
    if (Lb < qb)
      return fail(PA_ERR_INVALID_ARG, "seqlens_k[%d] = %d < new tokens %d (seqlens_k counts "
                  "every key, the new ones included)", b, Lb, qb);
    if (static_cast<int64_t>(Lb) > static_cast<int64_t>(p->max_blocks_per_seq) * bs)
      return fail(PA_ERR_INVALID_ARG, "seqlens_k[%d] = %d exceeds max_blocks_per_seq * "
                  "block_size = %d", b, Lb, p->max_blocks_per_seq * bs);
    if (qb > max_q) max_q = qb;  // exact max_query_len
    if (Lb > max_k) max_k = Lb;
    if (qb > 0) total_blocks += (Lb + bs - 1) / bs;
  }
  const int total_q = B > 0 ? cu_seqlens_q_host[B] : 0;
  p->total_q = total_q;
  p->max_query_len = max_q;
  p->max_seqlen_k = max_k;
  const int64_t max_rows = static_cast<int64_t>(max_q) * G;
  // Units with more rows than one mma.sync tile (16) go to the tensor-core
  // prefill kernel (items of one KV head and up to 64 rows) where it supports
  // the cache format; otherwise 4 rows (at most 4 per sequence and KV head: a
  // decode step with G <= 4), 8 or 16.
  const bool prefill = max_rows > 16 && pa::prefill_supported(p->kv_dtype, p->head_size, bs, B);
  p->rows_per_cta = prefill ? pa::prefill_rows_per_item()
                            : (max_rows > 8 ? 16 : (max_rows > 4 ? 8 : 4));
  p->num_row_groups = static_cast<int>((max_rows + p->rows_per_cta - 1) / p->rows_per_cta);
  const int sms = p->num_sms > 0 ? p->num_sms : current_sm_count();
  const int max_nblk = (max_k + bs - 1) / bs;
  // Split target T (KV blocks per split).  Automatic choice: the T that minimises
  // an estimate of the makespan of the work items over the resident CTAs:
  // (rounds - 1) * mean item + largest item + rounds * per-item cost + the split
  // partials' write and read spread over the CTAs + the combine kernel when
  // anything is split (flash decoding after the
  // GQA GEMV decode page, Code analysis 2, sized for the resident CTA slots).
  const int rows = p->rows_per_cta;
  const int HP = prefill ? 1 : pa::kHeadsPerItem;  // KV heads per item
  const int Hg = (p->kv_num_heads + HP - 1) / HP;  // head groups of one item each
  const double block_bytes = 2.0 * bs * cache_row_bytes(p->kv_dtype, p->head_size) *
                             (p->kv_num_heads < HP ? p->kv_num_heads : HP);
  const double item_cost = kItemCostBytes / block_bytes;
  const double part_cost = 2.0 * HP * rows * (p->head_size * 2.0 + 4.0) / block_bytes;
  const int64_t slots = static_cast<int64_t>(sms) *
                        (prefill ? 1 : pa::forward_ctas_per_sm(p->kv_dtype, p->head_size, bs, rows));
  auto count = [&](int T, int64_t* items, int64_t* split_items, int* max_bps, int* max_ns,
                   double* work) {
    *items = *split_items = 0;
    *max_bps = *max_ns = 0;
    *work = 0.0;
    for (int b = 0; b < B; ++b) {
      const int qb = cu_seqlens_q_host[b + 1] - cu_seqlens_q_host[b];
      if (qb == 0) continue;
      const int64_t units = static_cast<int64_t>(Hg) * ((static_cast<int64_t>(qb) * G + rows - 1) / rows);
      const int nblk = (seqlens_k_host[b] + bs - 1) / bs;
      int ns, bps;
      pa::split_geometry(nblk, T, kMaxSplits, &ns, &bps);
      *items += units * ns;
      if (ns > 1) *split_items += units * ns;
      if (bps > *max_bps) *max_bps = bps;
      if (ns > *max_ns) *max_ns = ns;
      *work += static_cast<double>(units) * nblk;
    }
  };
  int T = max_nblk > 0 ? max_nblk : 1;
  if (p->split_blocks > 0) {
    T = p->split_blocks;
  } else if (p->split_blocks == 0 && max_nblk > 1 && total_q > 0) {
    double best = -1.0;
    int prev_T = -1;
    for (int sp = 1; sp <= kMaxSplits && sp <= max_nblk; sp += (sp < 16 ? 1 : sp / 8)) {
      const int Tc = (max_nblk + sp - 1) / sp;
      if (Tc == prev_T) continue;
      prev_T = Tc;
      int64_t items, split_items;
      int max_bps, max_ns;
      double work;
      count(Tc, &items, &split_items, &max_bps, &max_ns, &work);
      if (items <= 0) break;
      const int64_t rounds = (items + slots - 1) / slots;
      // a split adds the combine kernel after the forward kernel
      const double est = (rounds - 1) * (work / items) + max_bps + rounds * item_cost +
                         split_items * part_cost / slots + (max_ns > 1 ? 2.0 * item_cost : 0.0);
      if (best < 0.0 || est < best) {
        best = est;
        T = Tc;
      }
    }
  }
  int64_t items = 0, split_items = 0;
  int max_bps = 0, max_ns = 1;
  double work = 0.0;
  count(T, &items, &split_items, &max_bps, &max_ns, &work);
  if (items >= (int64_t(1) << 31)) return fail(PA_ERR_UNSUPPORTED, "too many work items");
  p->blocks_per_split = T;
  p->num_splits = max_ns > 0 ? max_ns : 1;
  p->num_work_items = static_cast<int>(items);
  const size_t ws = ws_layout(p).total;
  p->workspace_bytes = ws;
  if (workspace_bytes_needed) *workspace_bytes_needed = ws;
  return ok();
}

pa_status paged_attn_forward(const void* q, const void* k_cache, const void* v_cache,
                             const float* k_scale, const float* v_scale,
                             const int32_t* block_table, const int32_t* seqlens_k,
                             const int32_t* cu_seqlens_q, void* out,
                             const paged_attn_params* p, void* stream) {
  pa_status st = check_problem(p);
  if (st != PA_OK) return st;
  if (p->total_q < 0 || p->max_query_len < 0)
    return fail(PA_ERR_INVALID_ARG, "params were not filled by paged_attn_plan");
  if (p->total_q == 0 || p->batch == 0 || p->max_query_len == 0) return ok();
  const bool prefill = p->rows_per_cta == pa::prefill_rows_per_item();
  if (p->rows_per_cta != 4 && p->rows_per_cta != 8 && p->rows_per_cta != 16 && !prefill)
    return fail(PA_ERR_INVALID_ARG, "params were not filled by paged_attn_plan (rows_per_cta)");
  if (prefill && !pa::prefill_supported(p->kv_dtype, p->head_size, p->block_size, p->batch))
    return fail(PA_ERR_INVALID_ARG, "params were not filled by paged_attn_plan (prefill kernel)");
  if (p->rows_per_cta == 4 && p->max_query_len * (p->num_heads / p->kv_num_heads) > 4)
    return fail(PA_ERR_INVALID_ARG, "params were not filled by paged_attn_plan (rows_per_cta)");
  if (p->num_splits > kMaxSplits)
    return fail(PA_ERR_INVALID_ARG, "num_splits %d exceeds %d", p->num_splits, kMaxSplits);
  const int G = p->num_heads / p->kv_num_heads;
  const int64_t need_rg = (static_cast<int64_t>(p->max_query_len) * G + p->rows_per_cta - 1) /
                          p->rows_per_cta;
  if (p->num_row_groups != need_rg || p->num_splits < 1 || p->blocks_per_split < 1 ||
      p->num_work_items < 0)
    return fail(PA_ERR_INVALID_ARG, "params were not filled by paged_attn_plan (grid)");
  if (!q || !k_cache || !v_cache || !k_scale || !v_scale || !block_table || !seqlens_k ||
      !cu_seqlens_q || !out)
    return fail(PA_ERR_INVALID_ARG, "a device pointer argument is NULL");
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16))
    return fail(PA_ERR_INVALID_ARG, "k_cache/v_cache must be 16-byte aligned (TMA)");
  if (!aligned(q, 16) || !aligned(k_scale, 16) || !aligned(v_scale, 16))
    return fail(PA_ERR_INVALID_ARG, "q, k_scale and v_scale must be 16-byte aligned (bulk copies)");
  if (!aligned(out, p->out_dtype == PA_F32 ? 16 : 4))
    return fail(PA_ERR_INVALID_ARG, "out must be 4-byte aligned (16-byte for PA_F32)");
  if (p->workspace == nullptr || p->workspace_bytes < kHeaderBytes)
    return fail(PA_ERR_WORKSPACE, "workspace missing (plan asks for %zu bytes)",
                p->workspace_bytes);
  if (!aligned(p->workspace, 256)) return fail(PA_ERR_WORKSPACE, "workspace not 256-aligned");
  if (p->num_blocks == 0) return fail(PA_ERR_INVALID_ARG, "num_blocks is 0 with keys to read");

  CUtensorMap kmap, vmap;
  const int box_heads = prefill ? 1 : pa::kHeadsPerItem;
  if ((st = encode_cache_map(k_cache, p, box_heads, &kmap)) != PA_OK) return st;
  if ((st = encode_cache_map(v_cache, p, box_heads, &vmap)) != PA_OK) return st;

  uint8_t* ws = static_cast<uint8_t*>(p->workspace);
  const WsLayout lay = ws_layout(p);
  if (lay.total > p->workspace_bytes)
    return fail(PA_ERR_WORKSPACE, "workspace_bytes %zu < %zu needed for %d splits",
                p->workspace_bytes, lay.total, p->num_splits);
  pa::FwdArgs a;
  a.q = q;
  a.out = out;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.block_table = block_table;
  a.seqlens_k = seqlens_k;
  a.cu_seqlens_q = cu_seqlens_q;
  a.err = reinterpret_cast<uint32_t*>(ws);
  a.work = reinterpret_cast<uint32_t*>(ws + pa::kWsWorkOffset);
  a.frag = reinterpret_cast<uint32_t*>(ws + lay.frag);
  a.o_part = p->num_splits > 1 ? reinterpret_cast<__half*>(ws + lay.o_part) : nullptr;
  a.lse_part = p->num_splits > 1 ? reinterpret_cast<float*>(ws + lay.lse_part) : nullptr;
  a.row_ns = p->num_splits > 1 ? reinterpret_cast<int32_t*>(ws + lay.row_ns) : nullptr;
  a.lse_out = p->lse_out;
  a.batch = p->batch;
  a.H = p->num_heads;
  a.Hk = p->kv_num_heads;
  a.G = G;
  a.maxb = p->max_blocks_per_seq;
  a.num_blocks = p->num_blocks;
  a.total_q = p->total_q;
  a.q_bf16 = p->q_dtype == PA_BF16;
  a.out_bf16 = p->out_dtype == PA_BF16;
  a.out_f32 = p->out_dtype == PA_F32;
  a.causal = p->causal;
  a.rows_cta = p->rows_per_cta;
  a.num_row_groups = p->num_row_groups;
  a.max_splits = p->num_splits;
  a.split_target = p->blocks_per_split;
  a.num_items = p->num_work_items;
  a.num_sms = p->num_sms > 0 ? p->num_sms : current_sm_count();
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale
                                             : 1.0f / sqrtf(static_cast<float>(p->head_size));
  a.sm_scale_log2 = scale * 1.4426950408889634f;
  a.stall_consumers = p->stall_consumers;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaEvent_t* ev = static_cast<cudaEvent_t*>(p->profile_events);
  cudaError_t e = cudaSuccess;
  if (ev != nullptr && (e = cudaEventRecord(ev[0], s)) != cudaSuccess)
    return cuda_status(e, "profile event record");
  e = prefill ? pa::launch_prefill(p->block_size, kmap, vmap, a, s)
              : pa::launch_forward(p->kv_dtype, p->head_size, p->block_size, p->rows_per_cta,
                                   kmap, vmap, a, s);
  if (e != cudaSuccess) return cuda_status(e, "forward launch");
  if (p->num_splits > 1) {
    e = pa::launch_combine(p->head_size, p->block_size, a, s);
    if (e != cudaSuccess) return cuda_status(e, "combine launch");
  }
  if (ev != nullptr && (e = cudaEventRecord(ev[1], s)) != cudaSuccess)
    return cuda_status(e, "profile event record");
  return ok();
}

pa_status paged_attn_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (workspace == nullptr || workspace_bytes == 0)
    return fail(PA_ERR_WORKSPACE, "workspace is NULL or empty");
  cudaError_t e =
      cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_status(e, "workspace memset");
  return ok();
}

pa_status paged_attn_read_device_error(void* workspace, int clear, uint32_t* bits, void* stream) {
  if (bits == nullptr) return fail(PA_ERR_INVALID_ARG, "bits is NULL");
  if (workspace == nullptr) {
    // the error word of paged_attn_forward_noalloc's scratch on this device
    const pa_status st = pa::noalloc_scratch_address(&workspace);
    if (st != PA_OK) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && clear) {
    e = cudaMemsetAsync(workspace, 0, sizeof(word), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  }
  if (e != cudaSuccess) return cuda_status(e, "reading the device error word");
  *bits = word;
  if (word & PA_DEVERR_BAD_BLOCK)
    return fail(PA_ERR_BAD_BLOCK_TABLE, "device error word 0x%x: block_table entry outside "
                "[0, num_blocks)", word);
  if (word)
    return fail(PA_ERR_DEVICE, "device error word 0x%x (2: wait timeout, 4: non-finite k_scale, "
                "8: device lengths contradict the plan)", word);
  return ok();
}

pa_status paged_kv_pack_int4(const int8_t* src, uint8_t* dst, int64_t rows, int head_size,
                             void* stream) {
  if (!src || !dst) return fail(PA_ERR_INVALID_ARG, "src/dst is NULL");
  if (rows < 0 || head_size <= 0 || head_size % 8 != 0)
    return fail(PA_ERR_INVALID_ARG, "rows >= 0 and head_size a positive multiple of 8 needed");
  if (!aligned(src, 8) || !aligned(dst, 4))
    return fail(PA_ERR_INVALID_ARG, "src must be 8-byte and dst 4-byte aligned");
  if (rows == 0) return ok();
  cudaError_t e =
      pa::launch_pack_int4(src, dst, rows, head_size, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_status(e, "pack_int4 launch");
}

pa_status paged_kv_unpack_int4(const uint8_t* src, int8_t* dst, int64_t rows, int head_size,
                               void* stream) {
  if (!src || !dst) return fail(PA_ERR_INVALID_ARG, "src/dst is NULL");
  if (rows < 0 || head_size <= 0 || head_size % 8 != 0)
    return fail(PA_ERR_INVALID_ARG, "rows >= 0 and head_size a positive multiple of 8 needed");
  if (!aligned(src, 4) || !aligned(dst, 8))
    return fail(PA_ERR_INVALID_ARG, "src must be 4-byte and dst 8-byte aligned");
  if (rows == 0) return ok();
  cudaError_t e =
      pa::launch_unpack_int4(src, dst, rows, head_size, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_status(e, "unpack_int4 launch");
}

pa_status paged_kv_gather_decode(const void* cache, const int32_t* block_table,
                                 const paged_attn_params* p, int b, int kv, int len_b,
                                 int dst_dtype, void* dst, void* stream) {
  pa_status st = check_problem(p);
  if (st != PA_OK) return st;
  if (!cache || !block_table || !dst) return fail(PA_ERR_INVALID_ARG, "NULL pointer argument");
  if (b < 0 || b >= p->batch || kv < 0 || kv >= p->kv_num_heads)
    return fail(PA_ERR_INVALID_ARG, "b=%d or kv=%d out of range", b, kv);
  if (len_b < 0 || static_cast<int64_t>(len_b) >
                       static_cast<int64_t>(p->max_blocks_per_seq) * p->block_size)
    return fail(PA_ERR_INVALID_ARG, "len_b=%d out of range", len_b);
  if (dst_dtype != PA_F16 && dst_dtype != PA_BF16)
    return fail(PA_ERR_INVALID_ARG, "dst_dtype must be PA_F16 or PA_BF16");
  if (!aligned(cache, 4)) return fail(PA_ERR_INVALID_ARG, "cache must be 4-byte aligned");
  if (len_b == 0) return ok();
  cudaError_t e = pa::launch_gather_decode(
      static_cast<const uint8_t*>(cache), block_table, p->kv_dtype, p->head_size, p->block_size,
      p->kv_num_heads, p->max_blocks_per_seq, p->num_blocks, b, kv, len_b, dst_dtype == PA_BF16,
      dst, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_status(e, "gather_decode launch");
}

pa_status paged_kv_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                          const float* k_scale, const float* v_scale, const int32_t* block_table,
                          const int32_t* seqlens_k, const int32_t* cu_seqlens_q,
                          const paged_attn_params* p, void* stream) {
  pa_status st = check_problem(p);
  if (st != PA_OK) return st;
  if (p->total_q < 0) return fail(PA_ERR_INVALID_ARG, "total_q %d < 0 (call paged_attn_plan)", p->total_q);
  if (p->total_q == 0 || p->batch == 0) return ok();
  if (!k_new || !v_new || !k_cache || !v_cache || !k_scale || !v_scale || !block_table ||
      !seqlens_k || !cu_seqlens_q)
    return fail(PA_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_scale, 16) ||
      !aligned(v_scale, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
    return fail(PA_ERR_INVALID_ARG, "new rows, scales and caches must be 16-byte aligned");
  if (p->workspace == nullptr || p->workspace_bytes < kHeaderBytes ||
      !aligned(p->workspace, 256))
    return fail(PA_ERR_WORKSPACE, "a 256-byte aligned workspace of >= 256 bytes holds the error word");
  if (static_cast<int64_t>(p->kv_num_heads) * p->head_size * 16 > 200 * 1024)
    return fail(PA_ERR_UNSUPPORTED, "kv_num_heads x head_size too large for the writer's "
                "shared-memory scales");
  pa::AppendArgs a;
  a.k_new = k_new;
  a.v_new = v_new;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.block_table = block_table;
  a.seqlens_k = seqlens_k;
  a.cu_seqlens_q = cu_seqlens_q;
  a.err = static_cast<uint32_t*>(p->workspace);
  a.batch = p->batch;
  a.Hk = p->kv_num_heads;
  a.maxb = p->max_blocks_per_seq;
  a.num_blocks = p->num_blocks;
  a.block_size = p->block_size;
  a.total_q = p->total_q;
  a.in_bf16 = p->q_dtype == PA_BF16;
  cudaError_t e = pa::launch_append(p->kv_dtype, p->head_size, a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_status(e, "append launch");
}

pa_status paged_attn_merge(const void* parts, int parts_dtype, const float* lse_parts,
                           int n_parts, int64_t rows, int head_size, void* out, int out_dtype,
                           float* lse_out, void* stream) {
  if (!parts || !lse_parts || !out) return fail(PA_ERR_INVALID_ARG, "NULL pointer argument");
  if (n_parts < 1 || n_parts > 64) return fail(PA_ERR_INVALID_ARG, "n_parts %d not in [1, 64]", n_parts);
  if (rows < 0) return fail(PA_ERR_INVALID_ARG, "rows < 0");
  if (head_size != 64 && head_size != 128)
    return fail(PA_ERR_UNSUPPORTED, "head_size %d not in {64, 128}", head_size);
  if (parts_dtype != PA_F16 && parts_dtype != PA_BF16 && parts_dtype != PA_F32)
    return fail(PA_ERR_INVALID_ARG, "parts_dtype must be PA_F16, PA_BF16 or PA_F32");
  if (out_dtype != PA_F16 && out_dtype != PA_BF16)
    return fail(PA_ERR_INVALID_ARG, "out_dtype must be PA_F16 or PA_BF16");
  if (!aligned(parts, parts_dtype == PA_F32 ? 16 : 8) || !aligned(out, 8) || !aligned(lse_parts, 4))
    return fail(PA_ERR_INVALID_ARG, "parts/out must be 8-byte (16 for fp32 parts) and lse_parts "
                "4-byte aligned");
  if (rows == 0) return ok();
  cudaError_t e = pa::launch_merge(parts, parts_dtype, lse_parts, n_parts, rows, head_size,
                                   out_dtype == PA_BF16, out, lse_out,
                                   static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_status(e, "merge launch");
}

pa_status paged_attn_stream_read(const void* src, size_t bytes, void* sink, void* stream) {
  if (!src || !sink) return fail(PA_ERR_INVALID_ARG, "src/sink is NULL");
  if (bytes % 16 != 0 || !aligned(src, 16) || !aligned(sink, 16))
    return fail(PA_ERR_INVALID_ARG, "bytes and pointers must be 16-byte multiples/aligned");
  cudaError_t e = pa::launch_stream_read(src, bytes, sink, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_status(e, "stream_read launch");
}

}  // extern "C"
