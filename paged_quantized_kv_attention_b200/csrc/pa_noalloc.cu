// pa_noalloc.cu -- paged_attn_forward_noalloc: the attention forward call with
// its workspace in a fixed device array owned by the library, for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where they
// run attention: code inside a CUDA-graph-replayed or otherwise frozen memory
// plan, plugins of a host framework that owns every device buffer and forbids
// allocation inside an operator, and real-time loops whose memory must be fixed
// at start-up.  They still hold the inputs and the output, but they cannot hand
// paged_attn_forward a workspace.  This entry point supplies one: the file-scope
// array below, PA_NOALLOC_MAX_WORKSPACE_BYTES long, which every GPU that loads
// this library holds until the process exits.
//
// The attention math, the kernels and the launch are exactly those of
// paged_attn_forward, which this function calls with the array's device address
// as the workspace.  It allocates nothing and frees nothing.
#include <stdarg.h>
#include <stdio.h>

#include "pa_internal.h"

namespace {

// The shared scratch.  In host code this name is only a host-side handle of the
// symbol, not a device address; the address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[PA_NOALLOC_MAX_WORKSPACE_BYTES];

// Records the message that paged_attn_last_error() returns on this thread.
pa_status noalloc_fail(pa_status st, const char* fmt, ...) {
  char msg[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(msg, sizeof(msg), fmt, ap);
  va_end(ap);
  return pa::set_last_error(st, msg);
}

}  // namespace

// Device address of the scratch on the current device.  Looked up on every call
// (a host-side query that allocates nothing): a cached address would dangle
// after the device's context is torn down and created again.  The first lookup
// on a device loads the library's device code there, which is why the first
// call should come before any stream capture.
pa_status pa::noalloc_scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr) {
    int dev = -1;
    cudaGetDevice(&dev);
    return noalloc_fail(PA_ERR_CUDA, "cudaGetSymbolAddress(scratch) on device %d: %s", dev,
                        cudaGetErrorString(e));
  }
  *out = p;
  return PA_OK;
}

extern "C" {

pa_status paged_attn_forward_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                     const float* k_scale, const float* v_scale,
                                     const int32_t* block_table, const int32_t* seqlens_k,
                                     const int32_t* cu_seqlens_q, void* out,
                                     const paged_attn_params* params, void* stream) {
  if (params == nullptr) return noalloc_fail(PA_ERR_INVALID_ARG, "params is NULL");
  const size_t need = params->workspace_bytes;
  if (need == 0)
    return noalloc_fail(PA_ERR_INVALID_ARG, "params were not filled by paged_attn_plan "
                        "(workspace_bytes is 0)");
  if (need > static_cast<size_t>(PA_NOALLOC_MAX_WORKSPACE_BYTES))
    return noalloc_fail(PA_ERR_WORKSPACE, "the plan needs %zu workspace bytes but the static "
                        "scratch of paged_attn_forward_noalloc holds %zu; plan again with "
                        "fewer KV splits (split_blocks) or use paged_attn_forward",
                        need, static_cast<size_t>(PA_NOALLOC_MAX_WORKSPACE_BYTES));
  if (params->total_q == 0 || params->batch == 0 || params->max_query_len == 0)
    return paged_attn_forward(q, k_cache, v_cache, k_scale, v_scale, block_table, seqlens_k,
                              cu_seqlens_q, out, params, stream);  // no launch, no scratch
  void* scratch = nullptr;
  pa_status st = pa::noalloc_scratch_address(&scratch);
  if (st != PA_OK) return st;

  // The array keeps the previous call's contents.  Zero what the kernel expects
  // to start at zero: the error word and the work counters (the header).  The
  // split partials are always written before they are read.
  size_t clear = pa::kWsHeaderBytes;
  if (clear > need) clear = need;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(scratch, 0, clear, s);
  if (e != cudaSuccess)
    return noalloc_fail(PA_ERR_CUDA, "clearing the static scratch: %s", cudaGetErrorString(e));

  paged_attn_params local = *params;
  local.workspace = scratch;
  local.workspace_bytes = need;
  st = paged_attn_forward(q, k_cache, v_cache, k_scale, v_scale, block_table, seqlens_k,
                          cu_seqlens_q, out, &local, stream);
  return st;  // paged_attn_forward has set the message of a failure
}

}  // extern "C"
