// pa_append.cu -- quantise-and-append: the cache write that precedes the
// attention call.  The new K and V rows of every sequence's new tokens are
// turned into per-channel symmetric codes (value = scale x code, the cache
// format of the INT4 paged-KV page, onnxruntime PR 32515, Code analysis 2-3)
// and stored at the slot the block table gives their absolute position.
//
// The code of a value is the code nearest to x / s, the quotient taken in IEEE
// single precision (one correctly rounded division), then INT8: nearest
// integer, ties to even, clamped to [-127, 127]; INT4: the same clamped to
// [-8, 7], channel 2j in the low nibble of byte j; FP8: round-to-nearest-even
// e4m3fn, saturating at +-448.  A NaN quotient stores 0 (integer caches) or
// 0x7F (FP8).
//
// HBM-bound and elementwise: a warp takes one new token's K and V rows; lane l
// handles 8-channel groups l, l + 32, ... of the token's Hk x D values (16 bytes
// of fp16/bf16 in, 8 or 4 bytes out), so both the reads and the row writes of a
// token (its heads are contiguous in the cache slot) are contiguous.  The
// per-channel scales and their rounded inverses sit in shared memory.
//
// Also here: the log-sum-exp merge of attention results over disjoint key sets
// (context parallelism; the flash-decoding combine of the GQA GEMV decode page,
// onnxruntime PR 29216, Code analysis 2).
#include <cuda_fp8.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

__device__ __forceinline__ float bits_to_float(uint32_t h, bool bf16) {
  return bf16 ? __uint_as_float(h << 16)
              : __half2float(__ushort_as_half(static_cast<unsigned short>(h)));
}

// Code of x under scale s (inv = RN(1 / s)): the code of the correctly rounded
// fp32 quotient x / s.  Integer caches: x * inv is within 2^-16 of x / s for
// |x / s| < 128 (two roundings of 2^-24 relative each), so its nearest integer
// is the code unless it lies within 2^-15 of a half-integer boundary (or on
// one); only then is the correctly rounded division taken.  Beyond the code
// range both forms clamp alike.  FP8: the correctly rounded division.
// The correctly rounded division, out of line: it runs only near a rounding
// boundary, and a call keeps it off the path of every other value.
__device__ __noinline__ float div_rn(float x, float s) { return __fdiv_rn(x, s); }

template <int KV>
__device__ __forceinline__ uint32_t code_of(float x, float s, float inv) {
  if constexpr (KV == PA_KV_FP8_E4M3) {
    const float q = __fdiv_rn(x, s);
    if (q != q) return 0x7Fu;
    return static_cast<uint32_t>(__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3)) & 0xFFu;
  } else {
    float q = __fmul_rn(x, inv);
    float r = rintf(q);
    if (__builtin_expect(fabsf(q - r) > 0.5f - 0x1p-15f, 0)) {
      q = div_rn(x, s);
      r = rintf(q);
    }
    // nearest integer, clamped (a NaN quotient converts to 0)
    constexpr int lo = KV == PA_KV_INT4 ? -8 : -127;
    constexpr int hi = KV == PA_KV_INT4 ? 7 : 127;
    const int c = min(max(__float2int_rn(r), lo), hi);
    return static_cast<uint32_t>(c) & (KV == PA_KV_INT4 ? 0xFu : 0xFFu);
  }
}

template <int KV>
__device__ __forceinline__ uint2 codes8(uint4 raw, float4 s0, float4 s1, float4 i0, float4 i1,
                                        bool bf16) {
  const float s[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};  // channel scales
  const float iv[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};  // their inverses
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t c[8];
#pragma unroll
  for (int e = 0; e < 8; ++e)
    c[e] = code_of<KV>(bits_to_float((w[e >> 1] >> (16 * (e & 1))) & 0xFFFFu, bf16), s[e], iv[e]);
  if constexpr (KV == PA_KV_INT4) {
    uint32_t out = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) out |= (c[2 * j] | (c[2 * j + 1] << 4)) << (8 * j);
    return make_uint2(out, 0u);
  } else {
    return make_uint2(c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24),
                      c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24));
  }
}

// One warp per new token, grid-striding over total_q: the warp decodes the
// token's sequence, position and page once, then its lanes walk the token's
// Hk x D/8 channel groups of K and of V together (16 input bytes each,
// contiguous across the lanes; all of a lane's loads go out before any code is
// computed).
template <int KV, int D>
__global__ void __launch_bounds__(256) pa_append_kernel(AppendArgs a) {
  constexpr int kGroups = D / 8;
  constexpr int kChs = KV == PA_KV_INT4 ? D / 2 : D;
  constexpr int kU = 4;  // groups per lane per pass (of K and of V)
  // scales of every channel, K then V, then their inverses: [2][2][Hk][D] fp32
  extern __shared__ float4 sc_s[];
  float* sc = reinterpret_cast<float*>(sc_s);
  const int n = a.Hk * D;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float ks = __ldg(a.k_scale + i), vs = __ldg(a.v_scale + i);
    sc[i] = ks;
    sc[n + i] = vs;
    sc[2 * n + i] = __frcp_rn(ks);  // the rounded inverses
    sc[3 * n + i] = __frcp_rn(vs);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int nwarps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  const int per_tok = a.Hk * kGroups;
  for (int tok = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
       tok < a.total_q; tok += nwarps) {
    // sequence of the token: the last b with cu[b] <= tok (warp-uniform)
    int lo = 0, hi = a.batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(a.cu_seqlens_q + mid) <= tok) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int q0 = __ldg(a.cu_seqlens_q + b), qb = __ldg(a.cu_seqlens_q + b + 1) - q0;
    const int Lb = __ldg(a.seqlens_k + b);
    if (qb <= 0 || qb > Lb || tok - q0 >= qb ||
        static_cast<long long>(Lb) > static_cast<long long>(a.maxb) * a.block_size) {
      if (lane == 0) record_error(a.err, PA_DEVERR_BAD_LENGTH);
      continue;
    }
    const int t = (Lb - qb) + (tok - q0);  // absolute position of the new token
    const int phys = __ldg(a.block_table + static_cast<size_t>(b) * a.maxb + t / a.block_size);
    if (phys < 0 || phys >= a.num_blocks) {
      if (lane == 0) record_error(a.err, PA_DEVERR_BAD_BLOCK);
      continue;  // the slot is unknown: nothing is written
    }
    const int slot = t % a.block_size;
    const size_t src_off = static_cast<size_t>(tok) * a.Hk * D;
    const uint4* ksrc = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.k_new) + src_off);
    const uint4* vsrc = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.v_new) + src_off);
    const size_t dst_off = (static_cast<size_t>(phys) * a.block_size + slot) * a.Hk * kChs;
    uint8_t* kdst = static_cast<uint8_t*>(a.k_cache) + dst_off;
    uint8_t* vdst = static_cast<uint8_t*>(a.v_cache) + dst_off;
    for (int g0 = 0; g0 < per_tok; g0 += 32 * kU) {
      uint4 kr[kU], vr[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int gi = g0 + 32 * u + lane;
        kr[u] = gi < per_tok ? __ldg(ksrc + gi) : make_uint4(0u, 0u, 0u, 0u);
        vr[u] = gi < per_tok ? __ldg(vsrc + gi) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int gi = g0 + 32 * u + lane;
        if (gi >= per_tok) break;
        // channels gi * 8 .. gi * 8 + 7 of the token's Hk x D row set
        const float4* ki = sc_s + 2 * gi;
        const float4* vi = sc_s + n / 4 + 2 * gi;
        const float4* kinv = sc_s + n / 2 + 2 * gi;
        const float4* vinv = sc_s + 3 * n / 4 + 2 * gi;
        const uint2 kc = codes8<KV>(kr[u], ki[0], ki[1], kinv[0], kinv[1], a.in_bf16);
        const uint2 vc = codes8<KV>(vr[u], vi[0], vi[1], vinv[0], vinv[1], a.in_bf16);
        // group gi is bytes [gi * 8, gi * 8 + 8) of the slot's Hk rows (INT4: 4)
        if constexpr (KV == PA_KV_INT4) {
          reinterpret_cast<uint32_t*>(kdst)[gi] = kc.x;
          reinterpret_cast<uint32_t*>(vdst)[gi] = vc.x;
        } else {
          reinterpret_cast<uint2*>(kdst)[gi] = kc;
          reinterpret_cast<uint2*>(vdst)[gi] = vc;
        }
      }
    }
  }
}

template <int KV, int D>
static cudaError_t launch_append_t(const AppendArgs& a, cudaStream_t stream) {
  if (a.total_q <= 0) return cudaSuccess;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long tasks = a.total_q;  // one warp per new token, 8 warps per CTA
  const long long want = (tasks + 7) / 8;
  const long long cap = static_cast<long long>(sms) * 8;  // 8 CTAs of 8 warps per SM
  const size_t smem = static_cast<size_t>(a.Hk) * D * 4 * sizeof(float);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(pa_append_kernel<KV, D>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  pa_append_kernel<KV, D><<<static_cast<unsigned>(want < cap ? want : cap), 256, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_append(int kv_dtype, int head_size, const AppendArgs& a, cudaStream_t stream) {
  const bool d128 = head_size == 128;
  switch (kv_dtype) {
    case PA_KV_INT8:
      return d128 ? launch_append_t<PA_KV_INT8, 128>(a, stream) : launch_append_t<PA_KV_INT8, 64>(a, stream);
    case PA_KV_INT4:
      return d128 ? launch_append_t<PA_KV_INT4, 128>(a, stream) : launch_append_t<PA_KV_INT4, 64>(a, stream);
    case PA_KV_FP8_E4M3:
      return d128 ? launch_append_t<PA_KV_FP8_E4M3, 128>(a, stream)
                  : launch_append_t<PA_KV_FP8_E4M3, 64>(a, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------------------
// Log-sum-exp merge of results over disjoint key sets: one warp per row; lane p
// holds part p's weight (n_parts <= 64: two per lane), then each lane sums its
// dims (a pair per step) over the parts in fp32.  PT: the parts' element type.
template <int D, int PT>
__global__ void __launch_bounds__(128) pa_merge_kernel(const void* __restrict__ parts,
                                                       const float* __restrict__ lse_parts,
                                                       int n_parts, long long rows, bool out_bf16,
                                                       uint16_t* __restrict__ out,
                                                       float* __restrict__ lse_out) {
  const int lane = threadIdx.x & 31;
  const long long r = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (r >= rows) return;
  float l0 = lane < n_parts ? __ldg(lse_parts + static_cast<long long>(lane) * rows + r) : -INFINITY;
  float l1 = lane + 32 < n_parts ? __ldg(lse_parts + static_cast<long long>(lane + 32) * rows + r)
                                 : -INFINITY;
  float M = fmaxf(l0, l1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float w0 = (l0 == -INFINITY) ? 0.f : __expf(l0 - M);
  const float w1 = (l1 == -INFINITY) ? 0.f : __expf(l1 - M);
  float sum = w0 + w1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  if (lse_out != nullptr && lane == 0) lse_out[r] = sum > 0.f ? M + __logf(sum) : -INFINITY;
  constexpr int kPairs = D / 2;  // element pairs per row
  for (int d2 = lane; d2 < kPairs; d2 += 32) {
    float ax = 0.f, ay = 0.f;
    for (int pidx = 0; pidx < n_parts; ++pidx) {
      const float wv = __shfl_sync(0xffffffffu, pidx < 32 ? w0 : w1, pidx & 31) * inv;
      if (wv == 0.f) continue;  // empty part: its values are not read
      const long long e = (static_cast<long long>(pidx) * rows + r) * D;  // row start, elements
      float x, y;
      if constexpr (PT == PA_F32) {
        const float2 v = __ldg(reinterpret_cast<const float2*>(static_cast<const float*>(parts) + e) + d2);
        x = v.x;
        y = v.y;
      } else {
        const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(parts) + e) + d2);
        if constexpr (PT == PA_BF16) {
          x = __uint_as_float(v << 16);
          y = __uint_as_float(v & 0xFFFF0000u);
        } else {
          x = __half2float(__ushort_as_half(v & 0xFFFFu));
          y = __half2float(__ushort_as_half(v >> 16));
        }
      }
      ax = fmaf(wv, x, ax);
      ay = fmaf(wv, y, ay);
    }
    uint32_t o;
    if (out_bf16) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(ax, ay);
      o = *reinterpret_cast<const uint32_t*>(&h);
    } else {
      const __half2 h = __floats2half2_rn(ax, ay);
      o = *reinterpret_cast<const uint32_t*>(&h);
    }
    reinterpret_cast<uint32_t*>(out + r * D)[d2] = o;
  }
}

template <int D>
static cudaError_t launch_merge_d(const void* parts, int parts_dtype, const float* lse_parts,
                                  int n_parts, long long rows, bool out_bf16, uint16_t* out,
                                  float* lse_out, unsigned blocks, cudaStream_t stream) {
  switch (parts_dtype) {
    case PA_F32:
      pa_merge_kernel<D, PA_F32><<<blocks, 128, 0, stream>>>(parts, lse_parts, n_parts, rows,
                                                             out_bf16, out, lse_out);
      break;
    case PA_BF16:
      pa_merge_kernel<D, PA_BF16><<<blocks, 128, 0, stream>>>(parts, lse_parts, n_parts, rows,
                                                              out_bf16, out, lse_out);
      break;
    default:
      pa_merge_kernel<D, PA_F16><<<blocks, 128, 0, stream>>>(parts, lse_parts, n_parts, rows,
                                                             out_bf16, out, lse_out);
  }
  return cudaGetLastError();
}

cudaError_t launch_merge(const void* parts, int parts_dtype, const float* lse_parts, int n_parts,
                         long long rows, int head_size, bool out_bf16, void* out, float* lse_out,
                         cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const long long blocks = (rows + 3) / 4;
  if (blocks >= (1ll << 31)) return cudaErrorInvalidValue;
  auto* op = static_cast<uint16_t*>(out);
  if (head_size == 128)
    return launch_merge_d<128>(parts, parts_dtype, lse_parts, n_parts, rows, out_bf16, op, lse_out,
                               static_cast<unsigned>(blocks), stream);
  return launch_merge_d<64>(parts, parts_dtype, lse_parts, n_parts, rows, out_bf16, op, lse_out,
                            static_cast<unsigned>(blocks), stream);
}

}  // namespace pa
