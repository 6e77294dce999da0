// pa_prefill.cu -- tensor-core (tcgen05 / TMEM) paged attention for work items
// with many query rows: ragged prefill and mixed prefill/decode batches over an
// INT8 cache, head_size 128.
//
// A work item is (sequence, pair of KV heads, group of 64 query rows, KV
// split).  The 64 rows of one head are its (new token, query head of the GQA
// group) pairs, row r = token r / G, query head h G + r % G; they are the M
// side of M = 64 tcgen05 MMAs, whose accumulators occupy half of each TMEM
// sub-partition, so the two heads of a pair fill the 128 lanes: head 0 in
// lanes 0-15 of every sub-partition, head 1 in lanes 16-31.
//
// Per CTA (one per SM, persistent, items from an atomic counter):
//   warp 0    producer: one TMA box per 16 keys and head (the paged gather:
//             block table -> physical block) for K and V, into a two-stage ring
//             of 64-key tiles;
//   warp 1    allocates TMEM and issues every MMA from one thread:
//               S_i = Qdigit_i K^T  (kind::i8, M 64, N 64 keys, K 128 channels;
//                                    three digit planes i, raw INT8 cache codes
//                                    straight from the TMA tile)
//               O  += P V            (kind::f16, M 64, N 128 dims, K 64 keys;
//                                    P fp16 from shared memory, V the fp16
//                                    repack of the codes)
//             the QK of tile j + 1 is issued before the PV of tile j;
//   warps 2-5 softmax: one thread per (head, row) = one TMEM lane.  At the
//             start of an item a thread folds k_scale into its query row
//             (normalised by the power of two of max|k_scale| and of its row)
//             and writes the row's three signed 8-bit digit planes; per tile
//             it reads its logits from TMEM, masks (causal, item range),
//             updates its running maximum (raised only when a logit exceeds it
//             by more than 2^8; the O row in TMEM is rescaled then), writes its
//             fp16 P row; at the end it normalises, applies the V scale and
//             stores its output row (or an fp16 split partial in code units
//             and its log2-sum-exp for the combine kernel);
//   warps 6-9 repack each V tile's codes to fp16 (exact) in shared memory in
//             the MN-major layout the PV MMA reads.
//
// Numerics follow the decode kernel: logits exact up to the digit split of
// the folded query (error <= 2^-21 of max|q'| sum|k|), fp32 accumulation, P
// in fp16 (<= 2^8), the V scale applied once at the end.
//
// Sources: INT8 codes kept raw and converted to FP16 for the tensor-core MMA
// with FP32 accumulation, and tensor cores for the prefill tiles (INT8-KV
// tensor-core page, onnxruntime PR 33707, Code analysis 1, "Why this is
// good"); low-precision KV repacked to a 16-bit type in shared memory for the
// prefill MMAs (FP8 KV-cache prefill repacking page, flashinfer PR 3485, Code
// analysis); the K scale folded into Q with a power-of-two normaliser (INT4
// paged-KV page, onnxruntime PR 32515, Code analysis 3); the causal mask,
// online softmax and flash-decoding split with a partials buffer (GQA GEMV
// decode page, onnxruntime PR 29216, Code analysis 1-2).
#include <math.h>

#include <atomic>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_tc.cuh"

namespace pa {

namespace {

constexpr uint32_t kFullMask = 0xffffffffu;

// Geometry (INT8 codes, head_size 128: one 128-byte row per key and head).
constexpr int kPfRows = 64;       // query rows per head per item (M of the MMAs)
constexpr int kPfHeads = 2;       // KV heads per item
constexpr int kPfD = 128;         // head size
constexpr int kPfTile = 64;       // keys per tile (N of QK, K of PV)
constexpr int kPfBox = 16;        // keys per TMA box
constexpr int kPfBoxes = kPfTile / kPfBox;
constexpr int kPfStages = 2;      // KV ring stages
constexpr int kPfMaxSeqs = 1024;  // sequences in the item table
constexpr int kPfWarps = 10;
constexpr int kPfThreads = kPfWarps * 32;

// Shared memory (bytes; every operand tile 1024-byte aligned).
constexpr int kHeadTile = kPfTile * kPfD;                // 8 KB: 64 keys (rows) x 128 B
constexpr int kQOff = 0;                                 // Q digit planes [3][2 heads] 8 KB
constexpr int kRingOff = kQOff + 3 * kPfHeads * kHeadTile;           // 48 KB
constexpr int kStageBytes = 2 * kPfHeads * kHeadTile;                // K then V, 32 KB
constexpr int kV16Off = kRingOff + kPfStages * kStageBytes;         // 112 KB
constexpr int kV16Head = 2 * kHeadTile;                  // 16 KB: fp16, 2 MN atoms of 8 KB
constexpr int kV16Buf = kPfHeads * kV16Head;             // 32 KB
constexpr int kPOff = kV16Off + 2 * kV16Buf;             // 176 KB
constexpr int kPHead = kPfRows * 128;                    // 8 KB: 64 rows x 64 fp16
constexpr int kPBuf = kPfHeads * kPHead;                 // 16 KB
constexpr int kBarOff = kPOff + 2 * kPBuf;               // 208 KB
constexpr int kNumBars = 24;
constexpr int kDescOff = kBarOff + kNumBars * 8;
constexpr int kScaleOff = kDescOff + 2 * 64;             // per item slot: the v_scale rows
constexpr int kScaleSlot = kPfHeads * kPfD * 4;          // of the pair's heads (1 KB)
constexpr int kCrowOff = kScaleOff + 2 * kScaleSlot;     // row logit multipliers [2 heads][64]
constexpr int kMiscOff = kCrowOff + kPfHeads * kPfRows * 4;  // TMEM base, abort flag, MMA item queue
constexpr int kTableOff = kMiscOff + 64;
constexpr int kPfSmemBytes = kTableOff + kPfMaxSeqs * 4;
static_assert(kPfSmemBytes <= 227 * 1024, "shared memory budget");

// One (sequence, KV head, row group) unit of query digits in the workspace,
// written by the pre-pass in the shared-memory image the MMAs read: three
// planes of 64 rows x 128 bytes (128-byte swizzle), then the 64 rows' logit
// multipliers (fp32).  Only the unit's valid rows are written and copied.
constexpr int kQUnitBytes = 3 * kPfRows * kPfD + kPfRows * 4;

// Barrier indices.
enum : int {
  kBKvFull = 0,    // [2] TMA bytes of a stage landed (tx count)
  kBKvEmpty = 2,   // [2] stage consumed: QK commit + 4 repack warps
  kBSFull = 4,     // [2] logits of a tile in TMEM (commit)
  kBSFree = 6,     // [2] softmax warps read the logits (4)
  kBPFull = 8,     // [2] P tile in shared memory (4)
  kBVFull = 10,    // [2] fp16 V tile in shared memory (4)
  kBPvDone = 12,   // [2] PV MMAs of a tile completed (commit)
  kBQFull = 14,    // an item's query digit planes and multipliers landed (tx count)
  kBQEmpty = 15,   // last QK of an item completed (commit) and the 4 softmax warps
                   // read their multipliers
  kBOFree = 16,    // epilogue read the O accumulator (4)
  kBItemFull = 17, // [2] descriptor published, the pair's scale rows landed (tx count)
  kBItemEmpty = 19,// [2] slot released by the 9 consumer warps (softmax: after the epilogue)
  kBFinal = 21,    // the MMA thread's final commit
};

// TMEM columns: O accumulator, then two logit buffers of three digit planes.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 0;
constexpr uint32_t kSCol0 = 128;  // buffer b at kSCol0 + b * 192, plane i at + i * 64

constexpr uint32_t kIdescQK = instr_desc(kAccS32, kFmtS8, kFmtS8, kMajorK, kMajorK, kPfTile, kPfRows);
constexpr uint32_t kIdescPV = instr_desc(kAccF32, kFmtF16, kFmtF16, kMajorK, kMajorMN, kPfD, kPfRows);

// One work item as published by the producer (64 bytes, like the decode kernel's).
struct PfItem {
  int valid;
  int b, hp, rg, split;
  int q0, row0, row_end, past, kbeg, kend;  // keys [kbeg, kend) of the item
  int Lb, nsplit, ntiles, pad0, pad1;
};
static_assert(sizeof(PfItem) == 64, "descriptor slot size");

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bounded wait that also gives up when another warp has aborted the CTA.
__device__ __forceinline__ bool pf_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                        uint32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait_suspend(bar, parity, kSuspendHintNs)) {
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      record_error(err, PA_DEVERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Items of sequence b: (KV head pairs) x (row groups) x (splits).
template <int BS>
__device__ __forceinline__ int pf_seq_items(const FwdArgs& a, int q0, int qb, int Lb, bool& bad) {
  bad = (q0 < 0 || qb < 0 || qb > Lb || q0 + qb > a.total_q ||
         static_cast<long long>(Lb) > static_cast<long long>(a.maxb) * BS);
  if (bad || qb == 0) return 0;
  const int rg = (qb * a.G + kPfRows - 1) / kPfRows;
  if (rg > a.num_row_groups) {
    bad = true;
    return 0;
  }
  int ns, bps;
  split_geometry((Lb + BS - 1) / BS, a.split_target, a.max_splits, &ns, &bps);
  return ((a.Hk + 1) / 2) * rg * ns;
}

// Item `local` of sequence b; false when it has no keys.
template <int BS>
__device__ __forceinline__ bool pf_decode_item(const FwdArgs& a, int b, int local, int q0, int qb,
                                               int Lb, PfItem& d) {
  d.valid = 0;
  const int R = qb * a.G;
  const int rg_n = (R + kPfRows - 1) / kPfRows;
  int ns, bps;
  split_geometry((Lb + BS - 1) / BS, a.split_target, a.max_splits, &ns, &bps);
  d.split = local % ns;
  const int rest = local / ns;
  d.rg = rest % rg_n;
  d.hp = rest / rg_n;
  d.b = b;
  d.row0 = d.rg * kPfRows;
  d.row_end = min(R, d.row0 + kPfRows);
  d.q0 = q0;
  d.Lb = Lb;
  d.past = Lb - qb;
  const int i_last = (d.row_end - 1) / a.G;
  const int kmax = a.causal ? d.past + i_last + 1 : Lb;  // keys seen by some row
  const int nblk = (kmax + BS - 1) / BS;
  d.nsplit = (nblk + bps - 1) / bps;
  const int blk_begin = d.split * bps;
  if (blk_begin >= nblk) return false;
  d.kbeg = blk_begin * BS;
  d.kend = min(min(nblk, blk_begin + bps) * BS, kmax);
  d.ntiles = (d.kend - d.kbeg + kPfTile - 1) / kPfTile;
  d.valid = 1;
  return true;
}

// int8 x 4 -> two fp16x2 with the exact code values (byte u = code + 128 placed
// in the mantissa of 1024 gives 1024 + u; subtract 1152).
__device__ __forceinline__ void i8x4_to_h2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t y = w ^ 0x80808080u;
  lo = i8x2_to_h2(y, 0x4140);
  hi = i8x2_to_h2(y, 0x4342);
}

// ---------------------------------------------------------------------------
// Query pre-pass: one CTA per (sequence, KV head, row group) unit, eight
// threads per row, each on 16 channels (one 16-byte chunk of every digit
// plane).  The row folds the head's k_scale into its query, normalised by the
// power of two of max|k_scale| over the head (e_kv) and of its own row (e_q),
// splits q'' = q' 2^(6 - e_q) (|q''| < 64) into signed 8-bit digits
// d0 + d1 2^-7 + d2 2^-14 and writes them, with the row's logit multiplier
// C = softmax_scale log2(e) 2^(e_kv + e_q) (capped at 2^90), to the workspace
// unit in the image the prefill kernel copies into shared memory.  It also
// flags non-finite K or V scales.  Launched before the prefill kernel, which
// waits for this grid before reading the workspace.
constexpr int kPrepThreadsPerRow = 8;
constexpr int kPrepThreads = kPfRows * kPrepThreadsPerRow;

__global__ void __launch_bounds__(kPrepThreads) pa_pf_prep_kernel(const FwdArgs a) {
  __shared__ float ks[kPfD];
  __shared__ float wmax[kPrepThreads / 32];
  __shared__ int bad_scale;
  // The prefill kernel is launched as this grid's programmatic dependent but is
  // released only when every CTA here has finished (no launch_dependents): its
  // CTAs would otherwise hold every SM's shared memory and registers while
  // waiting for this grid.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int u = blockIdx.x;  // ((b * Hk + h) * num_row_groups + rg)
  const int rg = u % a.num_row_groups;
  const int bh = u / a.num_row_groups;
  const int h = bh % a.Hk, b = bh / a.Hk;
  const int tid = threadIdx.x;
  const int q0 = __ldg(a.cu_seqlens_q + b), qb = __ldg(a.cu_seqlens_q + b + 1) - q0;
  const int Lb = __ldg(a.seqlens_k + b);
  if (qb <= 0 || qb > Lb || q0 < 0 || q0 + qb > a.total_q) return;  // CTA-uniform
  const int R = qb * a.G;
  if (rg * kPfRows >= R) return;  // CTA-uniform
  if (tid == 0) bad_scale = 0;
  __syncthreads();
  float mloc = 0.f;
  if (tid < kPfD) {
    const float kv = __ldg(a.k_scale + static_cast<size_t>(h) * kPfD + tid);
    const float vv = __ldg(a.v_scale + static_cast<size_t>(h) * kPfD + tid);
    ks[tid] = kv;
    mloc = fabsf(kv);
    if (!(isfinite(kv) && isfinite(vv))) bad_scale = 1;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(kFullMask, mloc, o));
  if ((tid & 31) == 0) wmax[tid >> 5] = mloc;
  __syncthreads();
  if (tid == 0 && bad_scale && rg == 0) record_error(a.err, PA_DEVERR_BAD_SCALE);
  float ksmax = 0.f;
#pragma unroll
  for (int w = 0; w < kPfD / 32; ++w) ksmax = fmaxf(ksmax, wmax[w]);
  const int r = tid / kPrepThreadsPerRow, c = tid % kPrepThreadsPerRow;  // row, 16-channel chunk
  const int ru = rg * kPfRows + r;
  const bool live = ru < R;  // the row's eight threads agree
  int e_kv = 0;
  (void)frexpf(ksmax, &e_kv);
  const float f_kv = ldexpf(1.f, -e_kv);
  const size_t orow = static_cast<size_t>(q0 + (live ? ru : 0) / a.G) * a.H + h * a.G + (live ? ru : 0) % a.G;
  const uint4* qr = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.q) + orow * kPfD) + 2 * c;
  uint4 qv[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
  if (live) {
    qv[0] = __ldg(qr);
    qv[1] = __ldg(qr + 1);
  }
  const bool qbf = a.q_bf16;
  float wv[16];
  float rmax = 0.f;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const uint32_t w = (&qv[e >> 3].x)[(e >> 1) & 3];
    const uint32_t bits = (w >> (16 * (e & 1))) & 0xFFFFu;
    const float x = qbf ? __uint_as_float(bits << 16)
                        : __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
    wv[e] = x * (ks[16 * c + e] * f_kv);
    rmax = fmaxf(rmax, fabsf(wv[e]));
  }
  // the row's eight threads are consecutive lanes
#pragma unroll
  for (int o = 1; o < kPrepThreadsPerRow; o <<= 1) rmax = fmaxf(rmax, __shfl_xor_sync(kFullMask, rmax, o));
  if (!live) return;
  int e_q = 0;
  (void)frexpf(rmax, &e_q);
  const float fq = ldexpf(1.f, 6 - e_q);
  uint32_t dg[3][4];
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    uint32_t b0 = 0u, b1 = 0u, b2 = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float v = wv[4 * wd + e] * fq;
      const float t0 = rintf(v);
      v = (v - t0) * 128.f;
      const float t1 = rintf(v);
      v = (v - t1) * 128.f;
      const float t2 = rintf(v);
      b0 |= (static_cast<uint32_t>(static_cast<int>(t0)) & 0xFFu) << (8 * e);
      b1 |= (static_cast<uint32_t>(static_cast<int>(t1)) & 0xFFu) << (8 * e);
      b2 |= (static_cast<uint32_t>(static_cast<int>(t2)) & 0xFFu) << (8 * e);
    }
    dg[0][wd] = b0;
    dg[1][wd] = b1;
    dg[2][wd] = b2;
  }
  uint8_t* unit = reinterpret_cast<uint8_t*>(a.frag) + static_cast<size_t>(u) * kQUnitBytes;
  const size_t off = r * kPfD + ((c ^ (r & 7)) << 4);  // 128-byte swizzle of row r
#pragma unroll
  for (int i = 0; i < 3; ++i)
    *reinterpret_cast<uint4*>(unit + i * kPfRows * kPfD + off) =
        make_uint4(dg[i][0], dg[i][1], dg[i][2], dg[i][3]);
  if (c == 0)
    reinterpret_cast<float*>(unit + 3 * kPfRows * kPfD)[r] =
        fminf(ldexpf(a.sm_scale_log2, e_kv + e_q), 0x1p90f);
}

template <int BS>
__global__ void __launch_bounds__(kPfThreads, 1)
    pa_prefill_kernel(const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const FwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0u) {
    if (threadIdx.x == 0) record_error(a.err, PA_DEVERR_BAD_LENGTH);
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  PfItem* descs = reinterpret_cast<PfItem*>(smem + kDescOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kMiscOff + 4);
  int* s_incl = reinterpret_cast<int*>(smem + kTableOff);
  const uint32_t sbase = smem_u32(smem);
  auto q_tile = [&](int i, int h) { return sbase + kQOff + (i * kPfHeads + h) * kHeadTile; };
  auto k_tile = [&](int s, int h) { return sbase + kRingOff + s * kStageBytes + h * kHeadTile; };
  auto v_tile = [&](int s, int h) {
    return sbase + kRingOff + s * kStageBytes + (kPfHeads + h) * kHeadTile;
  };
  auto v16_tile = [&](int buf, int h) { return sbase + kV16Off + buf * kV16Buf + h * kV16Head; };
  auto p_tile = [&](int buf, int h) { return sbase + kPOff + buf * kPBuf + h * kPHead; };

  // ---- set-up: barriers, TMEM (before the wait on the previous grid)
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBKvFull + s), 1);
      mbar_init(bar(kBKvEmpty + s), 1 + 4);
      mbar_init(bar(kBSFull + s), 1);
      mbar_init(bar(kBSFree + s), 4);
      mbar_init(bar(kBPFull + s), 4);
      mbar_init(bar(kBVFull + s), 4);
      mbar_init(bar(kBPvDone + s), 1);
      mbar_init(bar(kBItemFull + s), 1);
      mbar_init(bar(kBItemEmpty + s), 9);
    }
    mbar_init(bar(kBQFull), 1);
    mbar_init(bar(kBQEmpty), 1 + 4);
    mbar_init(bar(kBOFree), 4);
    mbar_init(bar(kBFinal), 1);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
  }
  if (warp == 1) {
    // One CTA per SM (shared memory), and no other kernel of this library
    // uses TMEM, so the allocation never has to wait.
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Inputs may come from the previous kernel in the stream (programmatic launch).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");

  if (warp == 0) {
    // ======================================================== producer
    const uint64_t policy = l2_evict_first_policy();
    // item table: inclusive item prefix per sequence
    int total = 0;
    {
      bool bad_any = false;
      const int nk = (a.batch + 31) >> 5;
      for (int k = 0; k < nk; ++k) {
        const int b = 32 * k + lane;
        int x = 0;
        if (b < a.batch) {
          const int q0 = __ldg(a.cu_seqlens_q + b);
          const int q1 = __ldg(a.cu_seqlens_q + b + 1);
          bool bad = false;
          x = pf_seq_items<BS>(a, q0, q1 - q0, __ldg(a.seqlens_k + b), bad);
          bad_any |= bad;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(kFullMask, x, o);
          if (lane >= o) x += y;
        }
        s_incl[b] = total + x;
        total += __shfl_sync(kFullMask, x, 31);
      }
      __syncwarp();
      if (bad_any) record_error(a.err, PA_DEVERR_BAD_LENGTH);
    }
    auto locate = [&](int w, PfItem& d) -> bool {
      d.valid = 0;
      const int nk = (a.batch + 31) >> 5;
      int fb = -1;
      for (int k = 0; k < nk && fb < 0; ++k) {
        const int b = 32 * k + lane;
        const unsigned m = __ballot_sync(kFullMask, b < a.batch && s_incl[b] > w);
        if (m != 0u) fb = 32 * k + __ffs(m) - 1;
      }
      if (fb < 0) return false;
      const int base = fb > 0 ? s_incl[fb - 1] : 0;
      const int q0 = __ldg(a.cu_seqlens_q + fb);
      const int qb = __ldg(a.cu_seqlens_q + fb + 1) - q0;
      return pf_decode_item<BS>(a, fb, w - base, q0, qb, __ldg(a.seqlens_k + fb), d);
    };
    int uses0 = 0, uses1 = 0;  // items published in slot 0 / 1
    int slot = 0;
    int g = 0;                 // tiles issued (stage s armed (g + 1 - s) / 2 times)
    int nq = 0;                // items whose query planes were loaded
    bool ok = true;
    int w = blockIdx.x;
    uint32_t w_pref = 0;
    if (lane == 0) w_pref = atomicAdd(a.work, 1u);
    auto next_index = [&]() {
      const int nxt = static_cast<int>(gridDim.x + __shfl_sync(kFullMask, w_pref, 0));
      if (lane == 0) w_pref = atomicAdd(a.work, 1u);
      return nxt;
    };
    while (ok) {
      PfItem d = {};
      while (w < total) {
        if (locate(w, d)) break;
        w = next_index();
      }
      if (lane == 0) {
        const int u = slot ? uses1 : uses0;
        if (u > 0 && !pf_wait(bar(kBItemEmpty + slot), (u - 1) & 1, abort_flag, a.err)) {
          ok = false;
        } else {
          descs[slot] = d;
          if (d.valid) {
            // the pair's v_scale rows travel with the descriptor
            const int nh = (2 * d.hp + 1 < a.Hk) ? 2 : 1;
            const uint32_t bytes = nh * kPfD * 4;
            mbar_arrive_expect_tx(bar(kBItemFull + slot), bytes);
            bulk_load(sbase + kScaleOff + slot * kScaleSlot,
                      a.v_scale + static_cast<size_t>(2 * d.hp) * kPfD, bytes, bar(kBItemFull + slot));
          } else {
            mbar_arrive(bar(kBItemFull + slot));
          }
        }
      }
      ok = __shfl_sync(kFullMask, ok, 0);
      if (slot) ++uses1; else ++uses0;
      if (!ok || !d.valid) break;
      const int32_t* bt = a.block_table + static_cast<size_t>(d.b) * a.maxb;
      const int hA = 2 * d.hp;
      const bool hBv = hA + 1 < a.Hk;
      // the item's query digit planes and row multipliers (from the pre-pass),
      // once the previous item's last QK has read the planes
      if (lane == 0) {
        if (nq > 0 && !pf_wait(bar(kBQEmpty), (nq - 1) & 1, abort_flag, a.err)) {
          ok = false;
        } else {
          const int nrows = d.row_end - d.row0;
          const uint32_t rbytes = nrows * kPfD;
          mbar_arrive_expect_tx(bar(kBQFull), (hBv ? 2 : 1) * (3 * rbytes + kPfRows * 4));
          for (int h = 0; h < (hBv ? 2 : 1); ++h) {
            const uint8_t* unit = reinterpret_cast<const uint8_t*>(a.frag) +
                                  ((static_cast<size_t>(d.b) * a.Hk + hA + h) * a.num_row_groups + d.rg) *
                                      kQUnitBytes;
            for (int i = 0; i < 3; ++i)
              bulk_load(q_tile(i, h), unit + i * kPfRows * kPfD, rbytes, bar(kBQFull));
            bulk_load(sbase + kCrowOff + h * kPfRows * 4, unit + 3 * kPfRows * kPfD, kPfRows * 4,
                      bar(kBQFull));
          }
        }
      }
      ++nq;
      ok = __shfl_sync(kFullMask, ok, 0);
      if (!ok) break;
      // The item's block-table entries are cached in registers, 256 at a time
      // (entry cbase + 32 j + lane in bte[j]), loaded while the ring drains, so
      // no tile waits for its block ids.
      const int blk0 = d.kbeg / BS;
      const int nblk = (d.kend - 1) / BS - blk0 + 1;
      constexpr int kCache = 8;
      int cbase = 0;
      int bte[kCache];
      auto fill = [&](int base) {
#pragma unroll
        for (int j = 0; j < kCache; ++j) {
          const int e = base + 32 * j + lane;
          bte[j] = e < nblk ? __ldg(bt + blk0 + e) : 0;
        }
      };
      fill(0);
      for (int t = 0; t < d.ntiles && ok; ++t, ++g) {
        const int st = g & 1;
        const int key0 = d.kbeg + t * kPfTile;
        const int rel0 = key0 / BS - blk0;  // first block of the tile, relative to the item
        if (rel0 + kPfBoxes - cbase > 32 * kCache) {
          cbase = rel0;
          fill(cbase);
        }
        if (g >= kPfStages) {
          if (lane == 0 && !pf_wait(bar(kBKvEmpty + st), ((g >> 1) - 1) & 1, abort_flag, a.err))
            ok = false;
          ok = __shfl_sync(kFullMask, ok, 0);
          if (!ok) break;
        }
        // lane u < 4: the 16-key box u of the tile
        const int key = key0 + kPfBox * lane;
        const bool load = lane < kPfBoxes && key < d.kend;
        const int ci = (lane < kPfBoxes ? key / BS - blk0 : rel0) - cbase;  // cached entry
        int ph = 0;
#pragma unroll
        for (int j = 0; j < kCache; ++j) {
          const int v = __shfl_sync(kFullMask, bte[j], ci & 31);
          if ((ci >> 5) == j) ph = v;
        }
        int tok = 0;
        if (load) {
          if (ph < 0 || ph >= a.num_blocks) {
            record_error(a.err, PA_DEVERR_BAD_BLOCK);
            ph = a.num_blocks;  // out-of-range box: zero fill, no fault
          }
          tok = ph * BS + key % BS;
        }
        const int nb = __popc(__ballot_sync(kFullMask, load));
        if (lane == 0)
          mbar_arrive_expect_tx(bar(kBKvFull + st), nb * kPfBox * kPfD * 2 * (hBv ? 2 : 1));
        __syncwarp();
        if (load) {
          const uint32_t off = lane * kPfBox * kPfD;
          tma_load_3d(k_tile(st, 0) + off, &kmap, bar(kBKvFull + st), 0, tok, hA, policy);
          tma_load_3d(v_tile(st, 0) + off, &vmap, bar(kBKvFull + st), 0, tok, hA, policy);
          if (hBv) {
            tma_load_3d(k_tile(st, 1) + off, &kmap, bar(kBKvFull + st), 0, tok, hA + 1, policy);
            tma_load_3d(v_tile(st, 1) + off, &vmap, bar(kBKvFull + st), 0, tok, hA + 1, policy);
          }
        }
      }
      slot ^= 1;
      w = next_index();
    }
    (void)__shfl_sync(kFullMask, w_pref, 0);
    // leave no copy in flight: wait for the last fill armed in each stage
    // (tiles 0, 2, 4, ... use stage 0, tiles 1, 3, ... stage 1)
    const int arms = (g + 1 - lane) / 2;
    if (lane < kPfStages && arms > 0) {
      const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
      if (!mbar_wait_until(bar(kBKvFull + lane), (arms - 1) & 1, deadline))
        record_error(a.err, PA_DEVERR_TIMEOUT);
    }
  } else if (warp == 1) {
    // ======================================================== MMA issue
    // One thread runs two cursors over the same sequence of items: the QK of
    // tile gq (needs its K tile, a free logit buffer and, at an item's first
    // tile, the item's query planes) and the PV of tile gp < gq (needs the P
    // and fp16 V tiles and, at an item's first tile, the O accumulator read by
    // the previous epilogue).  Each step issues whichever is ready, so the QK of
    // the next tiles runs while the softmax of the current one is still busy.
    // Nothing here blocks: the producer's progress depends on these MMAs.
    bool issued = false;
    if (lane == 0) {
      int uses0 = 0, uses1 = 0;  // items taken from slot 0 / 1
      int slot = 0;
      // items whose QK started, in order, for the PV cursor: (tiles, head pair)
      int2* fifo = reinterpret_cast<int2*>(smem + kMiscOff + 16);
      int f_head = 0, f_count = 0;
      int gq = 0, tq = 0, iq = 0;  // QK: global tile, tile in item, item index
      int gp = 0, tp = 0, ip = 0;  // PV: the same
      bool have_q = false, q_end = false;
      PfItem dq = {};
      uint64_t idle_since = 0;
      bool ok = true;
      const uint32_t wait_hint = 500;
      while (ok) {
        bool progress = false;
        if (!have_q && !q_end && f_count < 4 &&
            mbar_try_wait(bar(kBItemFull + slot), (slot ? uses1 : uses0) & 1)) {
          if (slot) ++uses1; else ++uses0;
          dq = descs[slot];
          mbar_arrive(bar(kBItemEmpty + slot));
          slot ^= 1;
          if (dq.valid) {
            have_q = true;
            tq = 0;
            fifo[(f_head + f_count) & 3] = make_int2(dq.ntiles, dq.hp);
            ++f_count;
          } else {
            q_end = true;
          }
          progress = true;
        }
        if (have_q) {
          const int st = gq & 1;
          const bool ready = mbar_try_wait(bar(kBKvFull + st), (gq >> 1) & 1) &&
                             (gq < 2 || mbar_try_wait(bar(kBSFree + st), ((gq >> 1) - 1) & 1)) &&
                             (tq > 0 || mbar_try_wait(bar(kBQFull), iq & 1));
          if (ready) {
            tc_fence_after();
            const int nh = (2 * dq.hp + 1 < a.Hk) ? 2 : 1;
            for (int h = 0; h < nh; ++h) {
              const uint32_t lanes = static_cast<uint32_t>(16 * h) << 16;
              const uint64_t bd = sdesc_sw128(k_tile(st, h), 16, 1024);
#pragma unroll
              for (int i = 0; i < 3; ++i) {
                const uint32_t dst = tmem + kSCol0 + st * 192 + i * 64 + lanes;
                const uint64_t ad = sdesc_sw128(q_tile(i, h), 16, 1024);
#pragma unroll
                for (int k = 0; k < kPfD / 32; ++k)
                  tc_mma_i8(dst, ad + 2 * k, bd + 2 * k, kIdescQK, k > 0 ? 1u : 0u);
              }
            }
            issued = true;
            tc_commit(bar(kBSFull + st));
            tc_commit(bar(kBKvEmpty + st));  // K consumed (the repack warps release V)
            ++gq;
            if (++tq == dq.ntiles) {
              tc_commit(bar(kBQEmpty));
              have_q = false;
              ++iq;
            }
            progress = true;
          }
        }
        if (f_count > 0 && gp < gq) {
          const int2 dp = fifo[f_head];  // (tiles, head pair)
          const int bf = gp & 1;
          const uint32_t ph = (gp >> 1) & 1;
          const bool ready = mbar_try_wait(bar(kBPFull + bf), ph) &&
                             mbar_try_wait(bar(kBVFull + bf), ph) &&
                             (tp > 0 || ip == 0 || mbar_try_wait(bar(kBOFree), (ip - 1) & 1));
          if (ready) {
            tc_fence_after();
            const int nh = (2 * dp.y + 1 < a.Hk) ? 2 : 1;
            for (int h = 0; h < nh; ++h) {
              const uint32_t dst = tmem + kOCol + (static_cast<uint32_t>(16 * h) << 16);
              const uint64_t ad = sdesc_sw128(p_tile(bf, h), 16, 1024);
              const uint64_t bd = sdesc_sw128(v16_tile(bf, h), kHeadTile, 1024);
#pragma unroll
              for (int k = 0; k < kPfTile / 16; ++k)  // 16 keys per MMA
                tc_mma_f16(dst, ad + 2 * k, bd + 128 * k, kIdescPV, (tp > 0 || k > 0) ? 1u : 0u);
            }
            tc_commit(bar(kBPvDone + bf));
            ++gp;
            if (++tp == dp.x) {
              tp = 0;
              ++ip;
              f_head = (f_head + 1) & 3;
              --f_count;
            }
            progress = true;
          }
        }
        if (q_end && f_count == 0) break;
        if (progress) {
          idle_since = 0;
        } else {
          const uint64_t now = global_timer_ns();
          if (idle_since == 0) idle_since = now;
          if (*abort_flag) break;
          if (now - idle_since > kWaitLimitNs) {
            *abort_flag = 1;
            record_error(a.err, PA_DEVERR_TIMEOUT);
            break;
          }
          // sleep on the event most likely next: the pending PV's P tile, else
          // the next QK's K tile
          if (f_count > 0 && gp < gq)
            (void)mbar_try_wait_suspend(bar(kBPFull + (gp & 1)), (gp >> 1) & 1, wait_hint);
          else if (have_q)
            (void)mbar_try_wait_suspend(bar(kBKvFull + (gq & 1)), (gq >> 1) & 1, wait_hint);
          else
            __nanosleep(200);
        }
      }
    }
    __syncwarp();
    // every MMA this thread issued has completed before the TMEM is freed
    if (lane == 0 && issued) {
      tc_commit(bar(kBFinal));
      const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
      if (!mbar_wait_until(bar(kBFinal), 0, deadline)) record_error(a.err, PA_DEVERR_TIMEOUT);
    }
  } else if (warp < 6) {
    // ======================================================== softmax / epilogue
    const int p = warp & 3;                 // TMEM sub-partition
    const int hsel = lane >> 4;             // head of the pair
    const int row = 16 * p + (lane & 15);   // row within the item's row group
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * p) << 16);  // this warp's lanes
    int uses0 = 0, uses1 = 0;  // items taken from slot 0 / 1
    int slot = 0;
    int g = 0;
    int items = 0;
    bool ok = true;
    const size_t stride = static_cast<size_t>(a.total_q) * a.H;
    while (ok) {
      if (!pf_wait(bar(kBItemFull + slot), (slot ? uses1 : uses0) & 1, abort_flag, a.err)) break;
      if (slot) ++uses1; else ++uses0;
      const PfItem d = descs[slot];
      const int dslot = slot;  // released after the epilogue (its scale rows are read there)
      slot ^= 1;
      if (!d.valid) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBItemEmpty + dslot));
        break;
      }
      const int h = 2 * d.hp + hsel;
      const int nrows = d.row_end - d.row0;
      const bool valid = h < a.Hk && row < nrows;
      const bool warp_any = __any_sync(kFullMask, valid);
      const int ru = d.row0 + row;                 // row of the (sequence, head) unit
      const int tok_i = valid ? ru / a.G : 0;      // new token of the row
      const size_t orow = static_cast<size_t>(d.q0 + tok_i) * a.H + h * a.G + (valid ? ru % a.G : 0);
      const int lim = min(a.causal ? d.past + tok_i + 1 : d.Lb, d.kend);  // keys < lim visible
      const float* vsc = reinterpret_cast<const float*>(smem + kScaleOff + dslot * kScaleSlot) +
                         hsel * kPfD;  // the V scale row of this thread's head

      // ---- the row's logit multiplier C (from the pre-pass):
      // logit (log2 units) = C 2^-6 (S0 + S1 2^-7 + S2 2^-14)
      float w1 = 0.f, w2 = 0.f;
      if (!__all_sync(kFullMask, pf_wait(bar(kBQFull), items & 1, abort_flag, a.err))) {
        ok = false;
        break;
      }
      {
        const float crow = valid ? reinterpret_cast<const float*>(smem + kCrowOff)[hsel * kPfRows + row] : 0.f;
        w1 = crow * (1.f / 8192.f);     // times (S0 * 128 + S1)
        w2 = crow * (1.f / 1048576.f);  // times S2
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBQEmpty));

      // ---- tiles
      float m_ref = -INFINITY, l_sum = 0.f;
      for (int t = 0; t < d.ntiles && ok; ++t, ++g) {
        const int bf = g & 1;
        if (!__all_sync(kFullMask, pf_wait(bar(kBSFull + bf), (g >> 1) & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int key0 = d.kbeg + t * kPfTile;
        const uint32_t ts = tl + kSCol0 + bf * 192;
        if (!warp_any) {
          // no row of this warp is live: only the barrier protocol
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(bar(kBSFree + bf));
            mbar_arrive(bar(kBPFull + bf));
          }
          continue;
        }
        // the row's 64 masked logits, read from the three digit planes (two
        // waits for twelve TMEM loads), and their maximum
        float x[kPfTile];
        float mx = -INFINITY;
#pragma unroll
        for (int cp = 0; cp < kPfTile / 32; ++cp) {
          uint32_t s0[32], s1[32], s2[32];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            tmem_ld16(ts + 32 * cp + 16 * hh, *reinterpret_cast<uint32_t(*)[16]>(&s0[16 * hh]));
            tmem_ld16(ts + 64 + 32 * cp + 16 * hh, *reinterpret_cast<uint32_t(*)[16]>(&s1[16 * hh]));
            tmem_ld16(ts + 128 + 32 * cp + 16 * hh, *reinterpret_cast<uint32_t(*)[16]>(&s2[16 * hh]));
          }
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float v = fmaf(__int2float_rn(static_cast<int>(s0[j]) * 128 + static_cast<int>(s1[j])),
                                 w1, __int2float_rn(static_cast<int>(s2[j])) * w2);
            x[32 * cp + j] = (key0 + 32 * cp + j < lim) ? v : -INFINITY;
            mx = fmaxf(mx, x[32 * cp + j]);
          }
        }
        // the logits are in registers: the S buffer may be refilled
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBSFree + bf));
        // running maximum, raised lazily (P <= 2^8 stays safe in fp16)
        const bool raise = valid && mx > -INFINITY && (m_ref == -INFINITY || mx > m_ref + 8.f);
        float alpha = 1.f;
        if (raise) {
          alpha = (m_ref == -INFINITY) ? 0.f : fast_exp2(m_ref - mx);
          m_ref = mx;
          l_sum *= alpha;
        }
        if (__any_sync(kFullMask, raise) && t > 0) {
          // the O rows hold this item's sums: rescale them once the previous
          // tile's PV has completed
          if (!__all_sync(kFullMask, pf_wait(bar(kBPvDone + (bf ^ 1)), ((g - 1) >> 1) & 1, abort_flag, a.err))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < kPfD / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(tl + kOCol + 16 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
            tmem_st16(tl + kOCol + 16 * c, o);
          }
          tmem_wait_st();
        }
        // the P buffer is free once the PV two tiles back has completed
        if (g >= 2 &&
            !__all_sync(kFullMask, pf_wait(bar(kBPvDone + bf), ((g >> 1) - 1) & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
        // P = 2^(x - m) in fp16, 8 keys (16 bytes) per store, and the row sum
        {
          const uint32_t pt = p_tile(bf, hsel) + row * 128;
          const bool live = m_ref != -INFINITY;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t pw[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float p0 = live ? fast_exp2(x[8 * c + 2 * j] - m_ref) : 0.f;
              const float p1 = live ? fast_exp2(x[8 * c + 2 * j + 1] - m_ref) : 0.f;
              // the row sum takes the fp32 values; P enters the PV product in
              // fp16 (relative rounding <= 2^-12 per weight)
              l_sum += p0 + p1;
              pw[j] = h22u(__floats2half2_rn(p0, p1));
            }
            if (valid)
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(pt + ((c ^ (row & 7)) << 4)),
                           "r"(pw[0]), "r"(pw[1]), "r"(pw[2]), "r"(pw[3])
                           : "memory");
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBPFull + bf));
      }
      if (!ok) break;

      // ---- epilogue: O / l, V scale, store (or the split partial)
      const int glast = g - 1;
      if (!__all_sync(kFullMask, pf_wait(bar(kBPvDone + (glast & 1)), (glast >> 1) & 1, abort_flag, a.err))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (warp_any) {
        const bool is_split = d.nsplit > 1;
        const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
        const size_t prow = static_cast<size_t>(d.split) * stride + orow;
#pragma unroll 1
        for (int c = 0; c < kPfD / 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tl + kOCol + 16 * c, o);
          tmem_wait_ld();
          if (!valid) continue;
          uint32_t packed[8];
          if (!is_split && a.out_f32) {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + orow * kPfD + 16 * c);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 vs = reinterpret_cast<const float4*>(vsc + 16 * c)[j];
              dst[j] = make_float4(__uint_as_float(o[4 * j]) * inv * vs.x,
                                   __uint_as_float(o[4 * j + 1]) * inv * vs.y,
                                   __uint_as_float(o[4 * j + 2]) * inv * vs.z,
                                   __uint_as_float(o[4 * j + 3]) * inv * vs.w);
            }
          } else if (!is_split) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float2 vs = reinterpret_cast<const float2*>(vsc + 16 * c)[j];
              const float o0 = __uint_as_float(o[2 * j]) * inv * vs.x;
              const float o1 = __uint_as_float(o[2 * j + 1]) * inv * vs.y;
              if (a.out_bf16) {
                const __nv_bfloat162 bb = __floats2bfloat162_rn(o0, o1);
                packed[j] = *reinterpret_cast<const uint32_t*>(&bb);
              } else {
                packed[j] = h22u(__floats2half2_rn(o0, o1));
              }
            }
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.out) + orow * kPfD + 16 * c);
            dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              packed[j] = h22u(__floats2half2_rn(__uint_as_float(o[2 * j]) * inv,
                                                 __uint_as_float(o[2 * j + 1]) * inv));
            uint4* dst = reinterpret_cast<uint4*>(a.o_part + prow * kPfD + 16 * c);
            dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
          }
        }
        if (valid) {
          if (is_split) {
            a.lse_part[prow] = (l_sum > 0.f) ? m_ref + __log2f(l_sum) : -INFINITY;
          } else if (a.lse_out != nullptr) {
            a.lse_out[orow] = (l_sum > 0.f) ? (m_ref + __log2f(l_sum)) * 0.6931471805599453f
                                            : -INFINITY;
          }
          if (a.row_ns != nullptr && d.split == 0) a.row_ns[orow] = d.nsplit;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(kBOFree));
        mbar_arrive(bar(kBItemEmpty + dslot));
      }
      ++items;
    }
  } else {
    // ======================================================== V repack
    const int tid = threadIdx.x - 6 * 32;  // 0..127
    int uses0 = 0, uses1 = 0;  // items taken from slot 0 / 1
    int slot = 0;
    int g = 0;
    bool ok = true;
    while (ok) {
      if (!pf_wait(bar(kBItemFull + slot), (slot ? uses1 : uses0) & 1, abort_flag, a.err)) break;
      if (slot) ++uses1; else ++uses0;
      const PfItem d = descs[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBItemEmpty + slot));
      slot ^= 1;
      if (!d.valid) break;
      const int nh = (2 * d.hp + 1 < a.Hk) ? 2 : 1;
      for (int t = 0; t < d.ntiles && ok; ++t, ++g) {
        const int st = g & 1;
        if (!__all_sync(kFullMask, pf_wait(bar(kBKvFull + st), (g >> 1) & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
        if (g >= 2 &&
            !__all_sync(kFullMask, pf_wait(bar(kBPvDone + st), ((g >> 1) - 1) & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
        // 2 heads x 64 keys x 8 chunks of 16 codes; chunk ci = tid + 128 u
#pragma unroll 2
        for (int u = 0; u < 8; ++u) {
          const int ci = tid + 128 * u;
          const int hs = ci >> 9, key = (ci >> 3) & 63, c = ci & 7;
          if (hs >= nh) continue;
          uint4 v;
          const uint32_t src = v_tile(st, hs) + key * 128 + ((c ^ (key & 7)) << 4);
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(src));
          uint32_t hw[8];
          i8x4_to_h2x2(v.x, hw[0], hw[1]);
          i8x4_to_h2x2(v.y, hw[2], hw[3]);
          i8x4_to_h2x2(v.z, hw[4], hw[5]);
          i8x4_to_h2x2(v.w, hw[6], hw[7]);
          // dims 16c .. 16c + 15 -> MN atom c / 4, 16-byte chunks 2 (c % 4) and + 1
          const uint32_t rowb = v16_tile(st, hs) + (c >> 2) * kHeadTile + (key >> 3) * 1024 + (key & 7) * 128;
          const int cc = 2 * (c & 3);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowb + ((cc ^ (key & 7)) << 4)),
                       "r"(hw[0]), "r"(hw[1]), "r"(hw[2]), "r"(hw[3])
                       : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowb + (((cc + 1) ^ (key & 7)) << 4)),
                       "r"(hw[4]), "r"(hw[5]), "r"(hw[6]), "r"(hw[7])
                       : "memory");
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(kBVFull + st));
          mbar_arrive(bar(kBKvEmpty + st));
        }
      }
    }
  }

  // ---- teardown: every role has left its loop; free TMEM, rewind the counters
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(a.work + 1, 1u) == gridDim.x - 1) {
      a.work[0] = 0u;
      a.work[1] = 0u;
    }
  }
}

template <int BS>
cudaError_t launch_prefill_t(const CUtensorMap& kmap, const CUtensorMap& vmap, const FwdArgs& a,
                             cudaStream_t stream) {
  static std::atomic<int> configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !configured[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(pa_prefill_kernel<BS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kPfSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev < 64) configured[dev].store(1, std::memory_order_release);
  }
  const int grid = a.num_items < a.num_sms ? a.num_items : a.num_sms;
  if (grid < 1) return cudaSuccess;
  const long long units = static_cast<long long>(a.batch) * a.Hk * a.num_row_groups;
  if (units >= (1ll << 31)) return cudaErrorInvalidValue;
  {
    // the query pre-pass, a programmatic dependent of whatever precedes it
    cudaLaunchConfig_t pc = {};
    pc.gridDim = dim3(static_cast<unsigned>(units));
    pc.blockDim = dim3(kPrepThreads);
    pc.stream = stream;
    cudaLaunchAttribute pattr[1];
    pattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pattr[0].val.programmaticStreamSerializationAllowed = 1;
    pc.attrs = pattr;
    pc.numAttrs = 1;
    e = cudaLaunchKernelEx(&pc, pa_pf_prep_kernel, a);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPfThreads);
  cfg.dynamicSmemBytes = kPfSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, pa_prefill_kernel<BS>, kmap, vmap, a);
}

}  // namespace

bool prefill_supported(int kv_dtype, int head_size, int block_size, int batch) {
  return kv_dtype == PA_KV_INT8 && head_size == kPfD && (block_size == 16 || block_size == 32) &&
         batch <= kPfMaxSeqs;
}

int prefill_rows_per_item() { return kPfRows; }

int prefill_unit_words() { return kQUnitBytes / 4; }

cudaError_t launch_prefill(int block_size, const CUtensorMap& kmap, const CUtensorMap& vmap,
                           const FwdArgs& a, cudaStream_t stream) {
  if (block_size == 16) return launch_prefill_t<16>(kmap, vmap, a, stream);
  if (block_size == 32) return launch_prefill_t<32>(kmap, vmap, a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pa
