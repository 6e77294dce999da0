// pa_tc.cuh -- sm_100a fifth-generation tensor-core primitives (tcgen05) used
// by the prefill kernel: tensor-memory (TMEM) allocation, shared-memory matrix
// descriptors, the instruction descriptor, single-thread MMA issue with
// completion on an mbarrier, and TMEM <-> register moves.
//
// Layout facts the kernel relies on (PTX ISA, tcgen05 chapter):
//  - A TMEM address is (lane << 16) | column.  A warp may only touch the 32
//    lanes of its sub-partition, lanes 32 (warp id % 4) .. + 31.
//  - An M = 64 accumulator of a cta_group::1 MMA occupies lanes 0-15 of each of
//    the four sub-partitions (row r in lane 32 (r / 16) + r % 16), column n in
//    column n; a second M = 64 accumulator can sit in the same columns at lane
//    offset 16.
//  - Shared-memory operands use the 128-byte swizzle: 8 rows of 128 bytes form
//    a 1024-byte atom, the 16-byte chunk index of each row XORed with the row
//    index (the same pattern a TMA copy with CU_TENSOR_MAP_SWIZZLE_128B writes).
//    K-major: rows are M (or N) indices, the 128 bytes run along K; the stride
//    between 8-row groups is the SBO field; a K step inside the atom advances
//    the start address.  MN-major: the 128 bytes run along M (or N), rows are K
//    indices; SBO is the stride between 8-row K groups, LBO the stride between
//    128-byte MN atoms.
#pragma once

#include <stdint.h>

namespace pa {

// ---------------------------------------------------------------- TMEM

// Allocate `ncols` TMEM columns (a power of two >= 32) for this CTA; the base
// address is written to shared memory at `dst`.  Warp-collective.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Ordering of tcgen05 operations around thread synchronisation (mbarriers,
// __syncthreads).
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Generic-proxy writes to shared memory become visible to the tensor cores
// (async proxy) that read them through descriptors.
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// The mbarrier at `bar` receives one arrival once every tcgen05 operation this
// thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// ---------------------------------------------------------------- descriptors

// Shared-memory matrix descriptor, 128-byte swizzle: start address, leading
// byte offset (LBO), stride byte offset (SBO), all in bytes.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version of sm_100
  d |= static_cast<uint64_t>(2) << 61;  // 128-byte swizzle
  return d;
}

// Instruction descriptor fields (kind::f16 and kind::i8).
constexpr uint32_t kFmtF16 = 0, kFmtS8 = 1;      // operand formats
constexpr uint32_t kAccF32 = 1, kAccS32 = 2;     // accumulator formats
constexpr uint32_t kMajorK = 0, kMajorMN = 1;

__host__ __device__ constexpr uint32_t instr_desc(uint32_t acc, uint32_t afmt, uint32_t bfmt, uint32_t amajor,
                              uint32_t bmajor, uint32_t n, uint32_t m) {
  return (acc << 4) | (afmt << 7) | (bfmt << 10) | (amajor << 15) | (bmajor << 16) |
         ((n >> 3) << 17) | ((m >> 4) << 24);
}

// ---------------------------------------------------------------- MMA

// D[tmem] (+)= A[smem] * B[smem]^T, signed 8-bit operands, 32-bit integer
// accumulators.  Issued by one thread.
__device__ __forceinline__ void tc_mma_i8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same with 16-bit floating-point operands and fp32 accumulators.
__device__ __forceinline__ void tc_mma_f16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ---------------------------------------------------------------- TMEM <-> registers

// 16 consecutive 32-bit columns of the warp's 32 lanes (one lane per thread).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

}  // namespace pa
