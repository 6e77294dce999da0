// pa_device.cuh -- sm_100a device primitives of the paged quantised-KV attention
// kernels: mbarriers with bounded waits, TMA tile loads, ldmatrix / movmatrix /
// mma.sync wrappers, and the exact code -> fp16 conversions of the three cache
// formats.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "paged_attn.h"

namespace pa {

// Upper bound of any single pipeline wait.  A correct kernel never gets near it;
// on expiry the kernel records PA_DEVERR_TIMEOUT and unwinds instead of hanging.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_error(uint32_t* err_word, uint32_t bits) {
  if (err_word != nullptr) atomicOr(err_word, bits);
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that lets the hardware suspend the thread for up to hint_ns while the
// phase is incomplete (it resumes as soon as the phase completes).
__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t bar, uint32_t parity,
                                                      uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

constexpr uint32_t kSuspendHintNs = 20000;

// Wait for the phase with the given parity to complete, for at most kWaitLimitNs.
// The thread sleeps in try_wait; the clock is read only after a failed suspend.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait_suspend(bar, parity, kSuspendHintNs)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// Same, against an absolute deadline shared by several waits.
__device__ __forceinline__ bool mbar_wait_until(uint32_t bar, uint32_t parity,
                                                uint64_t deadline_ns) {
  while (!mbar_try_wait_suspend(bar, parity, kSuspendHintNs)) {
    if (global_timer_ns() > deadline_ns) return false;
  }
  return true;
}

// ---------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// One 3-D tile (box fixed by the tensor map) into shared memory, completion
// counted in bytes on `bar`.  No multicast.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar), "l"(policy)
      : "memory");
}

// One bulk copy (global -> shared, 16-byte aligned, a multiple of 16 bytes)
// completing on an mbarrier.  No multicast.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Hint: bring the 128-byte line holding p into L2 (no fault for any address).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)));
}

// L2 policy for data that is read exactly once (the KV stream).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------- warp MMA

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// D = A(16x16, row) * B(16x8, col) + D, fp16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------- conversions

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ __half2 u2h2(uint32_t u) {
  __half2 h;
  *reinterpret_cast<uint32_t*>(&h) = u;
  return h;
}

__device__ __forceinline__ uint32_t h22u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// INT8: with y = bytes ^ 0x80 (so byte = code + 128), placing byte u in the low
// mantissa of 0x64xx gives the fp16 value 1024 + u exactly; subtracting 1152
// leaves the signed code.  `sel` picks which two bytes land in the two halves.
__device__ __forceinline__ uint32_t i8x2_to_h2(uint32_t y_biased, uint32_t sel) {
  const uint32_t h = prmt(y_biased, 0x64646464u, sel);
  return h22u(__hsub2(u2h2(h), u2h2(0x64806480u)));  // 0x6480 = 1152
}

// INT4, low nibbles of bytes 0 and 2: (x & 0x000F000F) holds the raw nibbles;
// XOR with 0x0008 biases the two's complement code by +8 and 0x6400 makes the
// half 1024 + code + 8; subtract 1032.
__device__ __forceinline__ uint32_t i4lo_to_h2(uint32_t x) {
  const uint32_t h = (x & 0x000F000Fu) ^ 0x64086408u;
  return h22u(__hsub2(u2h2(h), u2h2(0x64086408u)));  // 0x6408 = 1032
}

// INT4, high nibbles of bytes 0 and 2: the half is 1024 + 16 (code + 8);
// times 1/16 minus 72 gives the code, exactly, in one fused multiply-add.
__device__ __forceinline__ uint32_t i4hi_to_h2(uint32_t x) {
  const uint32_t h = (x & 0x00F000F0u) ^ 0x64806480u;
  return h22u(__hfma2(u2h2(h), u2h2(0x2C002C00u), u2h2(0xD480D480u)));  // 1/16, -72
}

// FP8 e4m3: the four codes of x -> two fp16x2 (bytes 0,1 -> lo; bytes 2,3 -> hi;
// the lower code of each pair lands in the lower half).
__device__ __forceinline__ void e4m3x4_to_h2x2(uint32_t x, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(x));
}

// INT4 -> u8 (code + 8) bytes: nibbles 0,2,4,6 of x (low nibble of each byte).
__device__ __forceinline__ uint32_t i4lo_to_u8x4(uint32_t x) { return (x & 0x0F0F0F0Fu) ^ 0x08080808u; }
// nibbles 1,3,5,7 of x (high nibble of each byte).
__device__ __forceinline__ uint32_t i4hi_to_u8x4(uint32_t x) {
  return ((x >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
}

// D = A(16x32, row) * B(32x8, col) + D with int8 operands and int32 accumulators;
// A is signed (s8) or unsigned (u8), B signed.
template <bool A_UNSIGNED>
__device__ __forceinline__ void imma_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                           uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (A_UNSIGNED) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

// Exact int -> float for |v| < 2^22 with an integer offset folded in:
// returns (float)(v - off) using the 1.5 * 2^23 magic number.
__device__ __forceinline__ float int_to_float_exact(int v, int magic_minus_off) {
  return __int_as_float(v + magic_minus_off) - 12582912.0f;
}

__device__ __forceinline__ uint32_t pack_f32x2_to_h2(float lo, float hi) {
  return h22u(__floats2half2_rn(lo, hi));
}

}  // namespace pa
