// pa_codec.cu -- INT4 pack/unpack, the gather-decode test hook and the HBM
// read-ceiling kernel.
//
// INT4 layout (INT4 paged-KV page, onnxruntime PR 32515, Code analysis 2): two
// 4-bit values per byte, channel 2j in the low nibble of byte j and channel 2j+1
// in the high nibble, 4-bit two's complement.
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// One thread packs 8 channels (4 output bytes) per iteration.
__global__ void pa_pack_int4_kernel(const int8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                    int64_t n_words) {
  for (int64_t w = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; w < n_words;
       w += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint2 in = reinterpret_cast<const uint2*>(src)[w];  // 8 int8 channels
    uint32_t out = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t word = j < 2 ? in.x : in.y;
      const uint32_t lo = (word >> (16 * (j & 1))) & 0xFu;
      const uint32_t hi = (word >> (16 * (j & 1) + 8)) & 0xFu;
      out |= (lo | (hi << 4)) << (8 * j);
    }
    reinterpret_cast<uint32_t*>(dst)[w] = out;
  }
}

// One thread unpacks 4 bytes (8 channels) per iteration with sign extension.
__global__ void pa_unpack_int4_kernel(const uint8_t* __restrict__ src, int8_t* __restrict__ dst,
                                      int64_t n_words) {
  for (int64_t w = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; w < n_words;
       w += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t x = reinterpret_cast<const uint32_t*>(src)[w];
    uint32_t o[2] = {0, 0};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int nib = static_cast<int>((x >> (4 * k)) & 0xFu);
      const int v = nib >= 8 ? nib - 16 : nib;
      o[k >> 2] |= (static_cast<uint32_t>(v) & 0xFFu) << (8 * (k & 3));
    }
    reinterpret_cast<uint2*>(dst)[w] = make_uint2(o[0], o[1]);
  }
}

// Decode one 4-byte word of a cache row with the attention kernel's conversion
// routines into its channels' fp16 bit patterns, in channel order.
template <int KV>
__device__ __forceinline__ void decode_word(uint32_t x, uint16_t* h, int& n) {
  if constexpr (KV == PA_KV_INT8) {
    const uint32_t y = x ^ 0x80808080u;
    const uint32_t p01 = i8x2_to_h2(y, 0x4140), p23 = i8x2_to_h2(y, 0x4342);
    h[0] = p01 & 0xFFFF; h[1] = p01 >> 16; h[2] = p23 & 0xFFFF; h[3] = p23 >> 16;
    n = 4;
  } else if constexpr (KV == PA_KV_FP8_E4M3) {
    uint32_t p01, p23;
    e4m3x4_to_h2x2(x, p01, p23);
    h[0] = p01 & 0xFFFF; h[1] = p01 >> 16; h[2] = p23 & 0xFFFF; h[3] = p23 >> 16;
    n = 4;
  } else {
    // (ch0, ch4), (ch1, ch5), (ch2, ch6), (ch3, ch7) -> channel order
    const uint32_t l0 = i4lo_to_h2(x), h0 = i4hi_to_h2(x);
    const uint32_t l1 = i4lo_to_h2(x >> 8), h1 = i4hi_to_h2(x >> 8);
    h[0] = l0 & 0xFFFF; h[4] = l0 >> 16; h[1] = h0 & 0xFFFF; h[5] = h0 >> 16;
    h[2] = l1 & 0xFFFF; h[6] = l1 >> 16; h[3] = h1 & 0xFFFF; h[7] = h1 >> 16;
    n = 8;
  }
}

template <int KV>
__global__ void pa_gather_decode_kernel(const uint8_t* __restrict__ cache,
                                        const int32_t* __restrict__ block_table, int head_size,
                                        int block_size, int kv_num_heads, int maxb,
                                        int num_blocks, int b, int kv, int len_b, int dst_bf16,
                                        void* dst, uint32_t* bad) {
  const int chs = KV == PA_KV_INT4 ? head_size / 2 : head_size;
  const int words = chs / 4;
  const int64_t total = static_cast<int64_t>(len_b) * words;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / words);
    const int wd = static_cast<int>(i % words);
    const int phys = block_table[static_cast<int64_t>(b) * maxb + t / block_size];
    uint32_t x = 0;
    if (phys >= 0 && phys < num_blocks) {
      const int64_t row = (static_cast<int64_t>(phys) * block_size + t % block_size) *
                              kv_num_heads + kv;
      x = reinterpret_cast<const uint32_t*>(cache + row * chs)[wd];
    } else if (bad != nullptr) {
      atomicOr(bad, PA_DEVERR_BAD_BLOCK);
    }
    uint16_t h[8];
    int n = 0;
    decode_word<KV>(x, h, n);
    const int64_t o = static_cast<int64_t>(t) * head_size + static_cast<int64_t>(wd) * n;
    for (int k = 0; k < n; ++k) {
      if (dst_bf16) {
        const float f = __half2float(__ushort_as_half(h[k]));
        reinterpret_cast<__nv_bfloat16*>(dst)[o + k] = __float2bfloat16_rn(f);
      } else {
        reinterpret_cast<uint16_t*>(dst)[o + k] = h[k];
      }
    }
  }
}

// Read-only streaming kernel: 16-byte non-allocating loads, XOR checksum per block.
__global__ void __launch_bounds__(256) pa_stream_read_kernel(const uint4* __restrict__ src,
                                                             int64_t n16, uint4* sink) {
  uint4 acc = make_uint4(0, 0, 0, 0);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(v[u].x), "=r"(v[u].y), "=r"(v[u].z), "=r"(v[u].w)
                   : "l"(src + i + u * stride));
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      acc.x ^= v[u].x; acc.y ^= v[u].y; acc.z ^= v[u].z; acc.w ^= v[u].w;
    }
  }
  for (; i < n16; i += stride) {
    const uint4 v = src[i];
    acc.x ^= v.x; acc.y ^= v.y; acc.z ^= v.z; acc.w ^= v.w;
  }
  // one checksum per block (warp 0 lane 0 after a warp reduction is enough to
  // keep the loads alive)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    acc.x ^= __shfl_xor_sync(0xffffffffu, acc.x, o);
    acc.y ^= __shfl_xor_sync(0xffffffffu, acc.y, o);
    acc.z ^= __shfl_xor_sync(0xffffffffu, acc.z, o);
    acc.w ^= __shfl_xor_sync(0xffffffffu, acc.w, o);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicXor(&sink[blockIdx.x].x, acc.x);
    atomicXor(&sink[blockIdx.x].y, acc.y);
    atomicXor(&sink[blockIdx.x].z, acc.z);
    atomicXor(&sink[blockIdx.x].w, acc.w);
  }
}

static int grid_for(int64_t work, int threads) {
  int64_t g = (work + threads - 1) / threads;
  if (g > 148 * 32) g = 148 * 32;
  return static_cast<int>(g < 1 ? 1 : g);
}

cudaError_t launch_pack_int4(const int8_t* src, uint8_t* dst, int64_t rows, int head_size,
                             cudaStream_t s) {
  const int64_t n_words = rows * head_size / 8;  // head_size is a multiple of 8
  pa_pack_int4_kernel<<<grid_for(n_words, 256), 256, 0, s>>>(src, dst, n_words);
  return cudaGetLastError();
}

cudaError_t launch_unpack_int4(const uint8_t* src, int8_t* dst, int64_t rows, int head_size,
                               cudaStream_t s) {
  const int64_t n_words = rows * head_size / 8;
  pa_unpack_int4_kernel<<<grid_for(n_words, 256), 256, 0, s>>>(src, dst, n_words);
  return cudaGetLastError();
}

cudaError_t launch_gather_decode(const uint8_t* cache, const int32_t* block_table, int kv_dtype,
                                 int head_size, int block_size, int kv_num_heads, int maxb,
                                 int num_blocks, int b, int kv, int len_b, int dst_bf16,
                                 void* dst, cudaStream_t s) {
  const int chs = kv_dtype == PA_KV_INT4 ? head_size / 2 : head_size;
  const int64_t work = static_cast<int64_t>(len_b) * (chs / 4);
  const int grid = grid_for(work, 128);
  switch (kv_dtype) {
    case PA_KV_INT8:
      pa_gather_decode_kernel<PA_KV_INT8><<<grid, 128, 0, s>>>(
          cache, block_table, head_size, block_size, kv_num_heads, maxb, num_blocks, b, kv,
          len_b, dst_bf16, dst, nullptr);
      break;
    case PA_KV_INT4:
      pa_gather_decode_kernel<PA_KV_INT4><<<grid, 128, 0, s>>>(
          cache, block_table, head_size, block_size, kv_num_heads, maxb, num_blocks, b, kv,
          len_b, dst_bf16, dst, nullptr);
      break;
    case PA_KV_FP8_E4M3:
      pa_gather_decode_kernel<PA_KV_FP8_E4M3><<<grid, 128, 0, s>>>(
          cache, block_table, head_size, block_size, kv_num_heads, maxb, num_blocks, b, kv,
          len_b, dst_bf16, dst, nullptr);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_stream_read(const void* src, size_t bytes, void* sink, cudaStream_t s) {
  const int64_t n16 = static_cast<int64_t>(bytes / 16);
  pa_stream_read_kernel<<<148 * 8, 256, 0, s>>>(reinterpret_cast<const uint4*>(src), n16,
                                                 reinterpret_cast<uint4*>(sink));
  return cudaGetLastError();
}

}  // namespace pa
