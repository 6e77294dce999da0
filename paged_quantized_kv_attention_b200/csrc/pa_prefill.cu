// pa_prefill.cu -- tensor-core (tcgen05 / TMEM) paged attention for work items
// with many query rows: ragged prefill and mixed prefill/decode batches over an
// INT8 cache, head_size 128.
//
// A work item is (sequence, KV head, group of up to 64 query rows, KV split).
// The rows of the item are its (new token, query head of the GQA group) pairs,
// row r = token r / G, query head h G + r % G, padded to R = 16, 32, 48 or 64.
// Keys are the M side of every MMA ("swap-AB"), 128 keys per tile, so no MMA
// runs at half height whatever R is:
//   S^T = K Qd^T   kind::i8, M 128 keys, N 3R (the three signed 8-bit digit
//                  planes of the folded query side by side), K 128 channels;
//                  raw INT8 cache codes straight from the TMA tile;
//   O^T += V^T P^T kind::f16, M 128 dims, N 64 rows, K 16 keys per MMA; V the
//                  exact fp16 repack of the codes, P^T fp16 from shared memory.
// In TMEM a thread of a warp owns one lane: one key of the logits, one dim of
// the output.
//
// Per CTA (one per SM, persistent, items from an atomic counter in
// longest-first order), 14 warps:
//   warp 0       producer: per item the descriptor and the head's V-scale row,
//                the query digit planes and row multipliers (written by the
//                pre-pass kernel), then per tile one TMA box per 16 keys (the
//                paged gather: block table -> physical block) for K and V into
//                a three-stage ring;
//   warp 1       allocates TMEM and issues every MMA from one thread: the QK of
//                tile j + 1 (double-buffered logits) while the softmax of tile
//                j runs, the PV of tile j once its P and fp16 V are in place;
//   warps 2, 3,
//   12, 13       V repack: codes -> fp16 (exact) in the MN-major layout the PV
//                MMA reads;
//   warps 4-7,   softmax, two groups of four warps (one per TMEM sub-partition,
//   8-11         so a group covers the 128 keys); group q owns the row chunks
//                q and q + 2 (16 rows each).  Per tile a thread combines its
//                key's three digit logits for its rows, masks (causal, item
//                range), takes each row's maximum over the warp's 32 keys by a
//                halving shuffle exchange (lane j ends with row j) and over the
//                group's four warps through shared memory, raises the row's
//                running maximum only when a logit exceeds it by more than a
//                factor 2^15 (then the row's O^T column and partial sums are
//                rescaled), and
//                writes its
//                key's fp16 P^T row; at the end the group sums its row totals,
//                normalises, applies the V scale and stores its rows (or an
//                fp16 split partial in code units and its log2-sum-exp for the
//                combine kernel).
//
// Numerics follow the decode kernel: logits exact up to the digit split of the
// folded query (error <= 2^-21 of max|q'| sum|k|), fp32 accumulation, P in
// fp16 (<= 2^15, below the fp16 maximum 65504), the V scale applied once at the
// end.
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

// Geometry (INT8 codes, head_size 128: one 128-byte row per key).
constexpr int kPfRows = 64;       // query rows per item at most (N side)
constexpr int kPfD = 128;         // head size
constexpr int kPfTile = 128;      // keys per tile (M of both MMAs' key side)
constexpr int kPfBox = 16;        // keys per TMA box
constexpr int kPfBoxes = kPfTile / kPfBox;
constexpr int kPfStages = 3;      // KV ring stages
constexpr int kPfMaxSeqs = 1024;  // sequences in the item table
constexpr int kPfWarps = 14;
constexpr int kPfThreads = kPfWarps * 32;
constexpr int kSmWarp0 = 4;       // softmax warps 4 .. 11
constexpr int kSmWarps = 8;
constexpr int kRepackWarps = 4;   // warps 2, 3, 12, 13

// Shared memory (bytes; every operand tile 1024-byte aligned).
constexpr int kQPlanesBytes = 3 * kPfRows * kPfD;          // 24 KB: three planes of <= 64 rows
constexpr int kQOff = 0;                                   // two query slots
constexpr int kTileBytes = kPfTile * kPfD;                 // 16 KB: 128 keys x 128 B
constexpr int kRingOff = kQOff + 2 * kQPlanesBytes;        // 48 KB
constexpr int kStageBytes = 2 * kTileBytes;                // K then V
constexpr int kV16Off = kRingOff + kPfStages * kStageBytes;  // 144 KB
constexpr int kV16Atom = kPfTile * 128;                    // 16 KB: one 64-dim MN atom, 128 keys
constexpr int kV16Bytes = 2 * kV16Atom;
constexpr int kPOff = kV16Off + kV16Bytes;                 // 176 KB
constexpr int kPBytes = kPfTile * 128;                     // 16 KB: 128 keys x 64 rows fp16
constexpr int kBarOff = kPOff + 2 * kPBytes;               // 208 KB
constexpr int kNumBars = 32;
constexpr int kDescOff = kBarOff + kNumBars * 8;
constexpr int kVScaleOff = kDescOff + 2 * 64;              // per descriptor slot: the V-scale row
constexpr int kCrowOff = kVScaleOff + 2 * kPfD * 4;        // per query slot: 64 row multipliers
constexpr int kRedOff = kCrowOff + 2 * kPfRows * 4;        // [2 groups][2 parities][4 warps][32]
constexpr int kRedLOff = kRedOff + 2 * 2 * 4 * 32 * 4;     // [2 groups][4 warps][32]
constexpr int kRowOff = kRedLOff + 2 * 4 * 32 * 4;         // per softmax warp: kRowArrays x [32]
constexpr int kRowArrays = 5;                              // m, m used, alpha / 1/l, w, out row
constexpr int kMiscOff = kRowOff + kSmWarps * kRowArrays * 32 * 4;  // TMEM base, abort, MMA queue
constexpr int kTableOff = kMiscOff + 64;                   // inclusive item prefix, in work order
constexpr int kPermOff = kTableOff + kPfMaxSeqs * 4;        // work order: sequence of position p
constexpr int kHistOff = kPermOff + kPfMaxSeqs * 2;         // counting-sort buckets
constexpr int kSortBuckets = 256;
constexpr int kPfSmemBytes = kHistOff + kSortBuckets * 4;
static_assert(kPfSmemBytes <= 227 * 1024, "shared memory budget");

// One (sequence, KV head, row group) unit of query digits in the workspace,
// written by the pre-pass in the shared-memory image the MMAs read: three
// planes of R rows x 128 bytes (128-byte swizzle, plane stride R x 128 bytes,
// R the unit's rows rounded up to 16), then at a fixed offset the 64 rows'
// logit multipliers (fp32).  Only the unit's valid rows are written.
constexpr int kQUnitBytes = kQPlanesBytes + kPfRows * 4;

// Barrier indices.
enum : int {
  kBKvFull = 0,     // [3] TMA bytes of a stage landed (tx count)
  kBKvEmpty = 3,    // [3] stage consumed: QK commit + the repack warps
  kBSFull = 6,      // [2] logits of a tile in TMEM (commit)
  kBSFree = 8,      // [2] softmax warps read the logits (8)
  kBPFull = 10,     // [2] P^T tile in shared memory (8)
  kBPvDone = 12,    // [2] PV MMAs of a tile completed (commit)
  kBQFull = 14,     // [2] an item's digit planes and row multipliers landed (tx count)
  kBQEmpty = 16,    // [2] the item's last QK completed (commit), softmax read the multipliers (8)
  kBItemFull = 18,  // [2] descriptor published, the head's V-scale row landed (tx count)
  kBItemEmpty = 20, // [2] slot released (MMA 1, repack 4, softmax 8 after the epilogue)
  kBVFull = 22,     // fp16 V tile in shared memory (repack warps)
  kBOFree = 23,     // epilogue read the O^T accumulator (8)
  kBFinal = 24,     // the MMA thread's final commit
  kBXch = 25,       // [2 groups][2] softmax group exchange steps (4 warps)
};

// TMEM columns: two logit buffers (three planes of R columns each), then O^T.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCols = 3 * kPfRows;  // buffer b at b * 192
constexpr uint32_t kOCol = 2 * kSCols;    // 384: O^T, 64 columns (rows)

constexpr uint32_t kIdescPV = instr_desc(kAccF32, kFmtF16, kFmtF16, kMajorMN, kMajorMN, kPfRows, kPfTile);

// One work item as published by the producer (64 bytes).
struct PfItem {
  int valid;
  int b, h, rg, split;
  int q0, row0, nrows, rpad, past, kbeg, kend;  // keys [kbeg, kend) of the item
  int Lb, nsplit, ntiles, pad0;
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

// Items of sequence b: (KV heads) x (row groups) x (splits).
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
  return a.Hk * rg * ns;
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
  d.h = rest / rg_n;
  d.b = b;
  d.row0 = d.rg * kPfRows;
  d.nrows = min(R - d.row0, kPfRows);
  d.rpad = (d.nrows + 15) & ~15;
  d.q0 = q0;
  d.Lb = Lb;
  d.past = Lb - qb;
  const int i_last = (d.row0 + d.nrows - 1) / a.G;
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
// plane), 16 rows per pass over the unit's valid rows.  The row folds the
// head's k_scale into its query, normalised by the power of two of max|k_scale|
// over the head (e_kv) and of its own row (e_q), splits q'' = q' 2^(6 - e_q)
// (|q''| < 64) into signed 8-bit digits d0 + d1 2^-7 + d2 2^-14 and writes
// them, with the row's logit multiplier C = softmax_scale log2(e) 2^(e_kv + e_q)
// (capped at 2^90), to the workspace unit in the image the prefill kernel
// copies into shared memory.  It also flags non-finite K or V scales.  Launched
// before the prefill kernel, which waits for this grid before reading the
// workspace.
constexpr int kPrepThreadsPerRow = 8;
constexpr int kPrepRowsPerPass = 16;
constexpr int kPrepThreads = kPrepRowsPerPass * kPrepThreadsPerRow;  // 128 = kPfD
constexpr int kPrepPasses = kPfRows / kPrepRowsPerPass;
static_assert(kPrepThreads == kPfD, "one K scale per thread");

__global__ void __launch_bounds__(kPrepThreads) pa_pf_prep_kernel(const FwdArgs a) {
  __shared__ float ks[kPfD];
  __shared__ float wmax[kPrepThreads / 32];
  __shared__ int bad_scale;
  // The prefill kernel, this grid's programmatic dependent, may start now: it
  // builds its work order while this grid runs and waits for the grid before
  // reading the digit units.
  asm volatile("griddepcontrol.launch_dependents;");
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
  const int nrows = min(R - rg * kPfRows, kPfRows);
  const int rpad = (nrows + 15) & ~15;
  const int npass = (nrows + kPrepRowsPerPass - 1) / kPrepRowsPerPass;
  const int rq = tid / kPrepThreadsPerRow, c = tid % kPrepThreadsPerRow;  // row in a pass, chunk
  // every pass's 16 channels, in flight while the head's K scales are reduced
  uint4 qv[kPrepPasses][2];
#pragma unroll
  for (int ps = 0; ps < kPrepPasses; ++ps) {
    const int r = kPrepRowsPerPass * ps + rq;
    qv[ps][0] = qv[ps][1] = make_uint4(0u, 0u, 0u, 0u);
    if (r < nrows) {
      const int ru = rg * kPfRows + r;
      const size_t orow = static_cast<size_t>(q0 + ru / a.G) * a.H + h * a.G + ru % a.G;
      const uint4* qr = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.q) + orow * kPfD) + 2 * c;
      qv[ps][0] = __ldg(qr);
      qv[ps][1] = __ldg(qr + 1);
    }
  }
  if (tid == 0) bad_scale = 0;
  __syncthreads();
  const float kv = __ldg(a.k_scale + static_cast<size_t>(h) * kPfD + tid);
  const float vv = __ldg(a.v_scale + static_cast<size_t>(h) * kPfD + tid);
  ks[tid] = kv;
  float mloc = fabsf(kv);
  if (!(isfinite(kv) && isfinite(vv))) bad_scale = 1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(kFullMask, mloc, o));
  if ((tid & 31) == 0) wmax[tid >> 5] = mloc;
  __syncthreads();
  if (tid == 0 && bad_scale && rg == 0) record_error(a.err, PA_DEVERR_BAD_SCALE);
  float ksmax = 0.f;
#pragma unroll
  for (int w = 0; w < kPfD / 32; ++w) ksmax = fmaxf(ksmax, wmax[w]);
  int e_kv = 0;
  (void)frexpf(ksmax, &e_kv);
  const float f_kv = ldexpf(1.f, -e_kv);
  const bool qbf = a.q_bf16;
  float ksc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) ksc[e] = ks[16 * c + e] * f_kv;
  uint8_t* unit = reinterpret_cast<uint8_t*>(a.frag) + static_cast<size_t>(u) * kQUnitBytes;
#pragma unroll
  for (int ps = 0; ps < kPrepPasses; ++ps) {
    if (ps >= npass) break;  // CTA-uniform
    const int r = kPrepRowsPerPass * ps + rq;
    float wv[16];
    float rmax = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint32_t w = (&qv[ps][e >> 3].x)[(e >> 1) & 3];
      const uint32_t bits = (w >> (16 * (e & 1))) & 0xFFFFu;
      const float x = qbf ? __uint_as_float(bits << 16)
                          : __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
      wv[e] = x * ksc[e];
      rmax = fmaxf(rmax, fabsf(wv[e]));
    }
    // the row's eight threads are consecutive lanes
#pragma unroll
    for (int o = 1; o < kPrepThreadsPerRow; o <<= 1) rmax = fmaxf(rmax, __shfl_xor_sync(kFullMask, rmax, o));
    if (r >= nrows) continue;
    int e_q = 0;
    (void)frexpf(rmax, &e_q);
    const float fq = ldexpf(1.f, 6 - e_q);
    // Digits by round-to-nearest-even through the 1.5 * 2^23 magic number: for
    // |v| < 2^22, v + 1.5 * 2^23 rounds v to an integer t whose two's-complement
    // low byte is the low byte of the sum's bit pattern, and v - t is exact.
    constexpr float kMagic = 12582912.0f;
    uint32_t dg[3][4];
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      uint32_t b0 = 0u, b1 = 0u, b2 = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = wv[4 * wd + e] * fq;
        const float a0 = v + kMagic;
        v = (v - (a0 - kMagic)) * 128.f;
        const float a1 = v + kMagic;
        v = (v - (a1 - kMagic)) * 128.f;
        const float a2 = v + kMagic;
        b0 |= (__float_as_uint(a0) & 0xFFu) << (8 * e);
        b1 |= (__float_as_uint(a1) & 0xFFu) << (8 * e);
        b2 |= (__float_as_uint(a2) & 0xFFu) << (8 * e);
      }
      dg[0][wd] = b0;
      dg[1][wd] = b1;
      dg[2][wd] = b2;
    }
    const size_t off = r * kPfD + ((c ^ (r & 7)) << 4);  // 128-byte swizzle of row r
#pragma unroll
    for (int i = 0; i < 3; ++i)
      *reinterpret_cast<uint4*>(unit + i * rpad * kPfD + off) = make_uint4(dg[i][0], dg[i][1], dg[i][2], dg[i][3]);
    if (c == 0)
      reinterpret_cast<float*>(unit + kQPlanesBytes)[r] = fminf(ldexpf(a.sm_scale_log2, e_kv + e_q), 0x1p90f);
  }
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
  auto q_slot = [&](int s) { return sbase + kQOff + s * kQPlanesBytes; };
  auto k_tile = [&](int st) { return sbase + kRingOff + st * kStageBytes; };
  auto v_tile = [&](int st) { return sbase + kRingOff + st * kStageBytes + kTileBytes; };
  const uint32_t v16 = sbase + kV16Off;
  auto p_buf = [&](int b) { return sbase + kPOff + b * kPBytes; };

  // ---- set-up: barriers, TMEM (before the wait on the previous grid)
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kPfStages; ++s) {
      mbar_init(bar(kBKvFull + s), 1);
      mbar_init(bar(kBKvEmpty + s), 1 + kRepackWarps);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBSFull + s), 1);
      mbar_init(bar(kBSFree + s), kSmWarps);
      mbar_init(bar(kBPFull + s), kSmWarps);
      mbar_init(bar(kBPvDone + s), 1);
      mbar_init(bar(kBQFull + s), 1);
      mbar_init(bar(kBQEmpty + s), 1 + kSmWarps);
      mbar_init(bar(kBItemFull + s), 1);
      mbar_init(bar(kBItemEmpty + s), 1 + kRepackWarps + kSmWarps);
    }
    mbar_init(bar(kBVFull), kRepackWarps);
    mbar_init(bar(kBOFree), kSmWarps);
    mbar_init(bar(kBFinal), 1);
    for (int i = 0; i < 4; ++i) mbar_init(bar(kBXch + i), 4);
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
  // This grid may start while the pre-pass (its programmatic primary) runs: the
  // set-up above and the producer's work order touch only inputs; every role
  // that reads the pre-pass's units, uses the work counter or writes results
  // waits for the primary first.
  asm volatile("griddepcontrol.launch_dependents;");

  if (warp == 0) {
    // ======================================================== producer
    const uint64_t policy = l2_evict_first_policy();
    // Work order: sequences by decreasing number of key tiles (a stable
    // counting sort, so every CTA derives the same order), longest first so
    // that the items pulled last are short; then the inclusive item prefix in
    // that order.
    int16_t* s_perm = reinterpret_cast<int16_t*>(smem + kPermOff);
    int* s_hist = reinterpret_cast<int*>(smem + kHistOff);
    const int nk = (a.batch + 31) >> 5;
    auto bucket = [&](int b) {  // kSortBuckets - 1 - min(tiles, kSortBuckets - 1)
      const int L = __ldg(a.seqlens_k + b);
      const int tiles = L > 0 ? (L + kPfTile - 1) / kPfTile : 0;
      return kSortBuckets - 1 - min(tiles, kSortBuckets - 1);
    };
    for (int i = lane; i < kSortBuckets; i += 32) s_hist[i] = 0;
    __syncwarp();
    for (int k = 0; k < nk; ++k) {
      const int b = 32 * k + lane;
      if (b < a.batch) atomicAdd(s_hist + bucket(b), 1);
    }
    __syncwarp();
    {
      // exclusive prefix of the buckets: lane owns buckets 8 lane .. 8 lane + 7
      int v[kSortBuckets / 32];
      int sum = 0;
#pragma unroll
      for (int i = 0; i < kSortBuckets / 32; ++i) {
        v[i] = s_hist[(kSortBuckets / 32) * lane + i];
        sum += v[i];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFullMask, incl, o);
        if (lane >= o) incl += y;
      }
      int run = incl - sum;
#pragma unroll
      for (int i = 0; i < kSortBuckets / 32; ++i) {
        s_hist[(kSortBuckets / 32) * lane + i] = run;
        run += v[i];
      }
    }
    __syncwarp();
    for (int k = 0; k < nk; ++k) {
      const int b = 32 * k + lane;
      const int key = b < a.batch ? bucket(b) : kSortBuckets + lane;  // padding lanes match only themselves
      const unsigned same = __match_any_sync(kFullMask, key);
      const int rank = __popc(same & ((1u << lane) - 1u));
      const int base = b < a.batch ? s_hist[key] : 0;
      __syncwarp();
      if (b < a.batch) {
        s_perm[base + rank] = static_cast<int16_t>(b);
        if (rank == 0) s_hist[key] = base + __popc(same);
      }
      __syncwarp();
    }
    int total = 0;
    {
      bool bad_any = false;
      for (int k = 0; k < nk; ++k) {
        const int pos = 32 * k + lane;
        int x = 0;
        if (pos < a.batch) {
          const int b = s_perm[pos];
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
        s_incl[pos] = total + x;
        total += __shfl_sync(kFullMask, x, 31);
      }
      __syncwarp();
      if (bad_any) record_error(a.err, PA_DEVERR_BAD_LENGTH);
    }
    auto locate = [&](int w, PfItem& d) -> bool {
      d.valid = 0;
      int fp = -1;
      for (int k = 0; k < nk && fp < 0; ++k) {
        const int pos = 32 * k + lane;
        const unsigned m = __ballot_sync(kFullMask, pos < a.batch && s_incl[pos] > w);
        if (m != 0u) fp = 32 * k + __ffs(m) - 1;
      }
      if (fp < 0) return false;
      const int base = fp > 0 ? s_incl[fp - 1] : 0;
      const int fb = s_perm[fp];
      const int q0 = __ldg(a.cu_seqlens_q + fb);
      const int qb = __ldg(a.cu_seqlens_q + fb + 1) - q0;
      return pf_decode_item<BS>(a, fb, w - base, q0, qb, __ldg(a.seqlens_k + fb), d);
    };
    asm volatile("griddepcontrol.wait;" ::: "memory");
    int uses0 = 0, uses1 = 0;  // descriptors published in slot 0 / 1
    int slot = 0;
    int g = 0;                 // tiles issued (stage s armed (g + 2 - s) / 3 times)
    int nq = 0;                // items whose query planes were loaded (slot i & 1)
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
            // the head's V-scale row travels with the descriptor
            mbar_arrive_expect_tx(bar(kBItemFull + slot), kPfD * 4);
            bulk_load(sbase + kVScaleOff + slot * kPfD * 4, a.v_scale + static_cast<size_t>(d.h) * kPfD,
                      kPfD * 4, bar(kBItemFull + slot));
          } else {
            mbar_arrive(bar(kBItemFull + slot));
          }
        }
      }
      ok = __shfl_sync(kFullMask, ok, 0);
      if (slot) ++uses1; else ++uses0;
      if (!ok || !d.valid) break;
      const int32_t* bt = a.block_table + static_cast<size_t>(d.b) * a.maxb;
      // the item's query digit planes and row multipliers (from the pre-pass),
      // once the item two back has released the slot
      const int qs = nq & 1;
      if (lane == 0) {
        if (nq >= 2 && !pf_wait(bar(kBQEmpty + qs), ((nq >> 1) - 1) & 1, abort_flag, a.err)) {
          ok = false;
        } else {
          const uint32_t pbytes = 3 * d.rpad * kPfD;
          const uint8_t* unit = reinterpret_cast<const uint8_t*>(a.frag) +
                                ((static_cast<size_t>(d.b) * a.Hk + d.h) * a.num_row_groups + d.rg) *
                                    kQUnitBytes;
          mbar_arrive_expect_tx(bar(kBQFull + qs), pbytes + kPfRows * 4);
          bulk_load(q_slot(qs), unit, pbytes, bar(kBQFull + qs));
          bulk_load(sbase + kCrowOff + qs * kPfRows * 4, unit + kQPlanesBytes, kPfRows * 4,
                    bar(kBQFull + qs));
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
        const int st = g % kPfStages;
        const int key0 = d.kbeg + t * kPfTile;
        const int rel0 = key0 / BS - blk0;  // first block of the tile, relative to the item
        if (rel0 + kPfBoxes - cbase > 32 * kCache) {
          cbase = rel0;
          fill(cbase);
        }
        if (g >= kPfStages) {
          if (lane == 0 &&
              !pf_wait(bar(kBKvEmpty + st), ((g / kPfStages) - 1) & 1, abort_flag, a.err))
            ok = false;
          ok = __shfl_sync(kFullMask, ok, 0);
          if (!ok) break;
        }
        // lane u < 8: the 16-key box u of the tile
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
        if (lane == 0) mbar_arrive_expect_tx(bar(kBKvFull + st), nb * kPfBox * kPfD * 2);
        __syncwarp();
        if (load) {
          const uint32_t off = lane * kPfBox * kPfD;
          tma_load_3d(k_tile(st) + off, &kmap, bar(kBKvFull + st), 0, tok, d.h, policy);
          tma_load_3d(v_tile(st) + off, &vmap, bar(kBKvFull + st), 0, tok, d.h, policy);
        }
      }
      slot ^= 1;
      w = next_index();
    }
    (void)__shfl_sync(kFullMask, w_pref, 0);
    // leave no copy in flight: wait for the last fill armed in each stage (tile
    // g' uses stage g' % 3), in each query slot (item i uses slot i % 2) and in
    // each descriptor slot
    const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
    bool drained = true;
    if (lane < kPfStages) {
      const int arms = (g + kPfStages - 1 - lane) / kPfStages;
      if (arms > 0) drained &= mbar_wait_until(bar(kBKvFull + lane), (arms - 1) & 1, deadline);
    }
    if (lane < 2) {
      const int arms = (nq + 1 - lane) / 2;
      if (arms > 0) drained &= mbar_wait_until(bar(kBQFull + lane), (arms - 1) & 1, deadline);
      const int u = lane ? uses1 : uses0;
      if (u > 0) drained &= mbar_wait_until(bar(kBItemFull + lane), (u - 1) & 1, deadline);
    }
    if (!drained) record_error(a.err, PA_DEVERR_TIMEOUT);
  } else if (warp == 1) {
    // ======================================================== MMA issue
    // One thread runs two cursors over the same sequence of items: the QK of
    // tile gq (needs its K tile, a free logit buffer and, at an item's first
    // tile, the item's query planes) and the PV of tile gp < gq (needs the P^T
    // and fp16 V tiles and, at an item's first tile, the O^T accumulator read
    // by the previous epilogue).  Each step issues whichever is ready, so the
    // QK of the next tile runs while the softmax of the current one is busy.
    // Nothing here blocks: the producer's progress depends on these MMAs.
    bool issued = false;
    if (lane == 0) {
      int uses0 = 0, uses1 = 0;  // items taken from descriptor slot 0 / 1
      int slot = 0;
      int* fifo = reinterpret_cast<int*>(smem + kMiscOff + 16);  // tiles of the items in flight
      int f_head = 0, f_count = 0;
      int gq = 0, tq = 0, iq = 0;  // QK: global tile, tile in item, item index
      int gp = 0, tp = 0, ip = 0;  // PV: the same
      bool have_q = false, q_end = false;
      int q_ntiles = 0;
      uint32_t q_idesc = 0;
      uint64_t idle_since = 0;
      const uint32_t wait_hint = 500;
      const uint64_t bd_v = sdesc_sw128(v16, kV16Atom, 1024);
      while (true) {
        bool progress = false;
        if (!have_q && !q_end && f_count < 8 &&
            mbar_try_wait(bar(kBItemFull + slot), (slot ? uses1 : uses0) & 1)) {
          if (slot) ++uses1; else ++uses0;
          const PfItem dq = descs[slot];
          mbar_arrive(bar(kBItemEmpty + slot));
          slot ^= 1;
          if (dq.valid) {
            have_q = true;
            tq = 0;
            q_ntiles = dq.ntiles;
            q_idesc = instr_desc(kAccS32, kFmtS8, kFmtS8, kMajorK, kMajorK, 3 * dq.rpad, kPfTile);
            fifo[(f_head + f_count) & 7] = dq.ntiles;
            ++f_count;
          } else {
            q_end = true;
          }
          progress = true;
        }
        if (have_q) {
          const int st = gq % kPfStages;
          const bool ready = mbar_try_wait(bar(kBKvFull + st), (gq / kPfStages) & 1) &&
                             (gq < 2 || mbar_try_wait(bar(kBSFree + (gq & 1)), ((gq >> 1) - 1) & 1)) &&
                             (tq > 0 || mbar_try_wait(bar(kBQFull + (iq & 1)), (iq >> 1) & 1));
          if (ready) {
            tc_fence_after();
            const uint32_t dst = tmem + (gq & 1) * kSCols;
            const uint64_t ad = sdesc_sw128(k_tile(st), 16, 1024);
            const uint64_t bd = sdesc_sw128(q_slot(iq & 1), 16, 1024);
#pragma unroll
            for (int k = 0; k < kPfD / 32; ++k)  // 32 channels per MMA
              tc_mma_i8(dst, ad + 2 * k, bd + 2 * k, q_idesc, k > 0 ? 1u : 0u);
            issued = true;
            tc_commit(bar(kBSFull + (gq & 1)));
            tc_commit(bar(kBKvEmpty + st));  // K consumed (the repack warps release V)
            ++gq;
            if (++tq == q_ntiles) {
              tc_commit(bar(kBQEmpty + (iq & 1)));
              have_q = false;
              ++iq;
            }
            progress = true;
          }
        }
        if (f_count > 0 && gp < gq) {
          const int ntp = fifo[f_head];
          const bool ready = mbar_try_wait(bar(kBPFull + (gp & 1)), (gp >> 1) & 1) &&
                             mbar_try_wait(bar(kBVFull), gp & 1) &&
                             (tp > 0 || ip == 0 || mbar_try_wait(bar(kBOFree), (ip - 1) & 1));
          if (ready) {
            tc_fence_after();
            const uint64_t bd_p = sdesc_sw128(p_buf(gp & 1), kPBytes, 1024);
#pragma unroll
            for (int k = 0; k < kPfTile / 16; ++k)  // 16 keys (2048 bytes) per MMA
              tc_mma_f16(tmem + kOCol, bd_v + 128 * k, bd_p + 128 * k, kIdescPV,
                         (tp > 0 || k > 0) ? 1u : 0u);
            tc_commit(bar(kBPvDone + (gp & 1)));
            ++gp;
            if (++tp == ntp) {
              tp = 0;
              ++ip;
              f_head = (f_head + 1) & 7;
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
            (void)mbar_try_wait_suspend(bar(kBKvFull + gq % kPfStages), (gq / kPfStages) & 1, wait_hint);
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
  } else if (warp >= kSmWarp0 && warp < kSmWarp0 + kSmWarps) {
    // ======================================================== softmax / epilogue
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int grp = (warp - kSmWarp0) >> 2;  // row chunks grp and grp + 2
    const int v = warp & 3;                  // TMEM sub-partition: keys (dims) 32 v .. 32 v + 31
    const int kl = 32 * v + lane;            // this thread's key of a tile, dim of the output
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * v) << 16);
    float* red = reinterpret_cast<float*>(smem + kRedOff) + grp * 256;    // [parity][warp][32]
    float* redl = reinterpret_cast<float*>(smem + kRedLOff) + grp * 128;  // [warp][32]
    // this warp's per-row arrays, row index j = lane (row 16 (grp + 2 (j / 16)) + j % 16)
    float* rw = reinterpret_cast<float*>(smem + kRowOff) + (warp - kSmWarp0) * kRowArrays * 32;
    float* r_m = rw;            // running maximum (log2 units)
    float* r_mu = rw + 32;      // the maximum used for P (0 while none)
    float* r_al = rw + 64;      // rescale factor of the tile; 1 / l in the epilogue
    float* r_w = rw + 96;       // logit multiplier C 2^-13
    int* r_orow = reinterpret_cast<int*>(rw + 128);  // output row (-1: padding)
    const uint32_t p_row = static_cast<uint32_t>(kl) * 128u;  // this key's P^T row
    const uint32_t p_sw = static_cast<uint32_t>(kl & 7);
    // Exchange step xs of the group's four warps (shared-memory writes before
    // it are visible to the group after it): alternating barriers, bounded.
    int xs = 0;
    auto exchange = [&]() -> bool {
      __syncwarp();
      const uint32_t xb = bar(kBXch + 2 * grp + (xs & 1));
      if (lane == 0) mbar_arrive(xb);
      const bool done = __all_sync(kFullMask, pf_wait(xb, (xs >> 1) & 1, abort_flag, a.err));
      ++xs;
      return done;
    };
    int uses0 = 0, uses1 = 0;  // items taken from descriptor slot 0 / 1
    int slot = 0;
    int g = 0;
    int items = 0;
    bool ok = true;
    const size_t stride = static_cast<size_t>(a.total_q) * a.H;
    while (ok) {
      if (!__all_sync(kFullMask, pf_wait(bar(kBItemFull + slot), (slot ? uses1 : uses0) & 1, abort_flag, a.err)))
        break;
      if (slot) ++uses1; else ++uses0;
      const PfItem d = descs[slot];
      const int dslot = slot;  // released after the epilogue (its V-scale row is read there)
      slot ^= 1;
      if (!d.valid) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBItemEmpty + dslot));
        break;
      }
      const int c0 = grp, c1 = grp + 2;
      const bool n0 = 16 * c0 < d.rpad, n1 = 16 * c1 < d.rpad;  // n1 implies n0
      const int qs = items & 1;
      if (!__all_sync(kFullMask, pf_wait(bar(kBQFull + qs), (items >> 1) & 1, abort_flag, a.err))) {
        ok = false;
        break;
      }
      {
        const int jr = 16 * (lane < 16 ? c0 : c1) + (lane & 15);  // row of index lane
        const bool live = (lane < 16 ? n0 : n1) && jr < d.nrows;
        const float crow = live ? reinterpret_cast<const float*>(smem + kCrowOff + qs * kPfRows * 4)[jr] : 0.f;
        r_w[lane] = crow * (1.f / 8192.f);
        r_m[lane] = -INFINITY;
        r_mu[lane] = 0.f;
        int orow = -1;
        if (live) {
          const int ru = d.row0 + jr;
          orow = (d.q0 + ru / a.G) * a.H + d.h * a.G + ru % a.G;
        }
        r_orow[lane] = orow;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBQEmpty + qs));
      const int G = a.G;
      float l[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) l[j] = 0.f;

      // ---- tiles
      for (int t = 0; t < d.ntiles && ok; ++t, ++g) {
        const int b = g & 1;
        if (!__all_sync(kFullMask, pf_wait(bar(kBSFull + b), (g >> 1) & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (!n0) {
          // no row of this group: only the barrier protocol
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBSFree + b));
          if (g >= 2 &&
              !__all_sync(kFullMask, pf_wait(bar(kBPvDone + b), ((g >> 1) - 1) & 1, abort_flag, a.err))) {
            ok = false;
            break;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBPFull + b));
          continue;
        }
        const int key0 = d.kbeg + t * kPfTile;
        const int key = key0 + kl;
        // the key's logits for the group's rows (x[j], row index j), from the
        // three digit planes of each 16-row chunk
        float x[32];
        const uint32_t ts = tl + b * kSCols;
#pragma unroll
        for (int jc = 0; jc < 2; ++jc) {
          if (jc == 1 && !n1) {
#pragma unroll
            for (int i = 0; i < 16; ++i) x[16 + i] = -INFINITY;
            continue;
          }
          const uint32_t col = 16 * (jc ? c1 : c0);
          uint32_t s0[16], s1[16], s2[16];
          tmem_ld16(ts + col, s0);
          tmem_ld16(ts + d.rpad + col, s1);
          tmem_ld16(ts + 2 * d.rpad + col, s2);
          tmem_wait_ld();
#pragma unroll
          for (int i4 = 0; i4 < 4; ++i4) {
            const float4 w4 = reinterpret_cast<const float4*>(r_w + 16 * jc)[i4];
            const float ww[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 4 * i4 + e;
              const float tsum = fmaf(__int2float_rn(static_cast<int>(s2[i])), 0x1p-7f,
                                      __int2float_rn(static_cast<int>(s0[i]) * 128 + static_cast<int>(s1[i])));
              x[16 * jc + i] = tsum * ww[e];
            }
          }
        }
        // the logits are in registers: the S buffer may be refilled
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBSFree + b));
        // mask: the key is visible to item rows r >= rmin (causal) below the
        // item's key range end
        const bool mask_tile = (key0 + kPfTile > d.kend) ||
                               (a.causal && key0 + kPfTile - 1 > d.past + d.row0 / G);
        if (mask_tile) {
          const int rmin = key >= d.kend ? (1 << 30) : (a.causal ? max(0, G * (key - d.past) - d.row0) : 0);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int r = 16 * ((j >> 4) ? c1 : c0) + (j & 15);
            if (r < rmin) x[j] = -INFINITY;
          }
        }
        // row maxima: over the warp's keys, then over the group's warps
        float* rp = red + (xs & 1) * 128;
        {
          // halving exchange: lane j ends with the warp's maximum of row j
          float hv[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) hv[j] = x[j];
#pragma unroll
          for (int s = 16; s >= 1; s >>= 1) {
            const bool up = (lane & s) != 0;
#pragma unroll
            for (int i = 0; i < s; ++i) {
              const float send = up ? hv[i] : hv[i + s];
              const float keep = up ? hv[i + s] : hv[i];
              hv[i] = fmaxf(keep, __shfl_xor_sync(kFullMask, send, s));
            }
          }
          rp[32 * v + lane] = hv[0];
        }
        if (!exchange()) {
          ok = false;
          break;
        }
        bool resc;
        {
          const float tmax = fmaxf(fmaxf(rp[lane], rp[32 + lane]), fmaxf(rp[64 + lane], rp[96 + lane]));
          const float m_old = r_m[lane];
          const bool raise = tmax > m_old + 15.f;  // any visible logit when none yet
          const float m_new = raise ? tmax : m_old;
          r_m[lane] = m_new;
          r_mu[lane] = (m_new == -INFINITY) ? 0.f : m_new;
          r_al[lane] = raise ? fast_exp2(m_old - m_new) : 1.f;
          // the same in every warp of the group: the O^T columns and row sums
          // hold earlier tiles' terms of a raised row
          resc = __any_sync(kFullMask, raise && m_old != -INFINITY);
        }
        __syncwarp();
        if (resc) {
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4) {
            const float4 a4 = reinterpret_cast<const float4*>(r_al)[j4];
            l[4 * j4] *= a4.x;
            l[4 * j4 + 1] *= a4.y;
            l[4 * j4 + 2] *= a4.z;
            l[4 * j4 + 3] *= a4.w;
          }
          // the O^T columns of the group's rows, once the previous tile's PV has
          // completed (this warp's lanes: dims 32 v .. 32 v + 31)
          if (!__all_sync(kFullMask, pf_wait(bar(kBPvDone + (b ^ 1)), ((g - 1) >> 1) & 1, abort_flag, a.err))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int jc = 0; jc < 2; ++jc) {
            if (jc == 1 && !n1) continue;
            const uint32_t oc = tl + kOCol + 16 * (jc ? c1 : c0);
            uint32_t o[16];
            tmem_ld16(oc, o);
            tmem_wait_ld();
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) {
              const float4 a4 = reinterpret_cast<const float4*>(r_al + 16 * jc)[i4];
              o[4 * i4] = __float_as_uint(__uint_as_float(o[4 * i4]) * a4.x);
              o[4 * i4 + 1] = __float_as_uint(__uint_as_float(o[4 * i4 + 1]) * a4.y);
              o[4 * i4 + 2] = __float_as_uint(__uint_as_float(o[4 * i4 + 2]) * a4.z);
              o[4 * i4 + 3] = __float_as_uint(__uint_as_float(o[4 * i4 + 3]) * a4.w);
            }
            tmem_st16(oc, o);
          }
          tmem_wait_st();
        }
        // the P^T buffer is free once the PV two tiles back has completed
        if (g >= 2 &&
            !__all_sync(kFullMask, pf_wait(bar(kBPvDone + b), ((g >> 1) - 1) & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
        // P = 2^(x - m) in fp16 (8 rows, 16 bytes per store) and the row sums
        {
          const uint32_t pr = p_buf(b) + p_row;
#pragma unroll
          for (int jc = 0; jc < 2; ++jc) {
            if (jc == 1 && !n1) continue;
            const int c = jc ? c1 : c0;
            uint32_t pw[8];
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) {
              const float4 m4 = reinterpret_cast<const float4*>(r_mu + 16 * jc)[i4];
              const int j = 16 * jc + 4 * i4;
              const float p0 = fast_exp2(x[j] - m4.x);
              const float p1 = fast_exp2(x[j + 1] - m4.y);
              const float p2 = fast_exp2(x[j + 2] - m4.z);
              const float p3 = fast_exp2(x[j + 3] - m4.w);
              // the row sums take the fp32 values; P enters the PV product in
              // fp16 (relative rounding <= 2^-12 per weight)
              l[j] += p0;
              l[j + 1] += p1;
              l[j + 2] += p2;
              l[j + 3] += p3;
              pw[2 * i4] = h22u(__floats2half2_rn(p0, p1));
              pw[2 * i4 + 1] = h22u(__floats2half2_rn(p2, p3));
            }
            const uint32_t ch = static_cast<uint32_t>(2 * c);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(pr + ((ch ^ p_sw) << 4)),
                         "r"(pw[0]), "r"(pw[1]), "r"(pw[2]), "r"(pw[3])
                         : "memory");
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(pr + (((ch + 1) ^ p_sw) << 4)),
                         "r"(pw[4]), "r"(pw[5]), "r"(pw[6]), "r"(pw[7])
                         : "memory");
          }
        }
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBPFull + b));
      }
      if (!ok) break;

      // ---- epilogue: O / l, V scale, store (or the split partial)
      const int glast = g - 1;
      if (!__all_sync(kFullMask, pf_wait(bar(kBPvDone + (glast & 1)), (glast >> 1) & 1, abort_flag, a.err))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (n0) {
        // row sums over the warp's keys: halving exchange, lane j ends with row j
#pragma unroll
        for (int s = 16; s >= 1; s >>= 1) {
          const bool up = (lane & s) != 0;
#pragma unroll
          for (int i = 0; i < s; ++i) {
            const float send = up ? l[i] : l[i + s];
            const float keep = up ? l[i + s] : l[i];
            l[i] = keep + __shfl_xor_sync(kFullMask, send, s);
          }
        }
        redl[32 * v + lane] = l[0];
        if (!exchange()) {
          ok = false;
          break;
        }
        const float L = (redl[lane] + redl[32 + lane]) + (redl[64 + lane] + redl[96 + lane]);
        const float m = r_m[lane];
        const int orow_j = r_orow[lane];
        const bool is_split = d.nsplit > 1;
        r_al[lane] = L > 0.f ? 1.f / L : 0.f;
        if (v == 0 && orow_j >= 0) {
          const float lse2 = L > 0.f ? m + __log2f(L) : -INFINITY;
          if (is_split) {
            a.lse_part[static_cast<size_t>(d.split) * stride + orow_j] = lse2;
            if (d.split == 0 && a.row_ns != nullptr) a.row_ns[orow_j] = d.nsplit;
          } else {
            if (a.lse_out != nullptr) a.lse_out[orow_j] = lse2 * 0.6931471805599453f;
          }
        }
        __syncwarp();
        const float vs = reinterpret_cast<const float*>(smem + kVScaleOff + dslot * kPfD * 4)[kl];
#pragma unroll 1
        for (int jc = 0; jc < 2; ++jc) {
          if (jc == 1 && !n1) continue;
          uint32_t o[16];
          tmem_ld16(tl + kOCol + 16 * (jc ? c1 : c0), o);
          tmem_wait_ld();
#pragma unroll
          for (int i4 = 0; i4 < 4; ++i4) {
            const float4 inv4 = reinterpret_cast<const float4*>(r_al + 16 * jc)[i4];
            const int4 or4 = reinterpret_cast<const int4*>(r_orow + 16 * jc)[i4];
            const float iv[4] = {inv4.x, inv4.y, inv4.z, inv4.w};
            const int orr[4] = {or4.x, or4.y, or4.z, or4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if (orr[e] < 0) continue;
              const float val = __uint_as_float(o[4 * i4 + e]) * iv[e];
              const size_t orow = static_cast<size_t>(orr[e]);
              if (is_split) {
                a.o_part[(static_cast<size_t>(d.split) * stride + orow) * kPfD + kl] = __float2half_rn(val);
              } else if (a.out_f32) {
                reinterpret_cast<float*>(a.out)[orow * kPfD + kl] = val * vs;
              } else if (a.out_bf16) {
                reinterpret_cast<__nv_bfloat16*>(a.out)[orow * kPfD + kl] = __float2bfloat16_rn(val * vs);
              } else {
                reinterpret_cast<__half*>(a.out)[orow * kPfD + kl] = __float2half_rn(val * vs);
              }
            }
          }
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
    const int rw = (warp < 4) ? warp - 2 : warp - 10;  // 0..3
    const int tid = 32 * rw + lane;                     // 0..127
    int uses0 = 0, uses1 = 0;  // items taken from descriptor slot 0 / 1
    int slot = 0;
    int g = 0;
    bool ok = true;
    while (ok) {
      if (!__all_sync(kFullMask, pf_wait(bar(kBItemFull + slot), (slot ? uses1 : uses0) & 1, abort_flag, a.err)))
        break;
      if (slot) ++uses1; else ++uses0;
      const PfItem d = descs[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBItemEmpty + slot));
      slot ^= 1;
      if (!d.valid) break;
      for (int t = 0; t < d.ntiles && ok; ++t, ++g) {
        const int st = g % kPfStages;
        if (!__all_sync(kFullMask, pf_wait(bar(kBKvFull + st), (g / kPfStages) & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
        // the fp16 V buffer is free once the previous tile's PV has completed
        if (g >= 1 &&
            !__all_sync(kFullMask, pf_wait(bar(kBPvDone + ((g - 1) & 1)), ((g - 1) >> 1) & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
        // 128 keys x 8 chunks of 16 codes; chunk ci = tid + 128 u
#pragma unroll 4
        for (int u = 0; u < 8; ++u) {
          const int ci = tid + 128 * u;
          const int key = ci >> 3, c = ci & 7;
          uint4 vv;
          const uint32_t src = v_tile(st) + key * 128 + ((c ^ (key & 7)) << 4);
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(vv.x), "=r"(vv.y), "=r"(vv.z), "=r"(vv.w)
                       : "r"(src));
          uint32_t hw[8];
          i8x4_to_h2x2(vv.x, hw[0], hw[1]);
          i8x4_to_h2x2(vv.y, hw[2], hw[3]);
          i8x4_to_h2x2(vv.z, hw[4], hw[5]);
          i8x4_to_h2x2(vv.w, hw[6], hw[7]);
          // dims 16c .. 16c + 15 -> MN atom c / 4, 16-byte chunks 2 (c % 4) and + 1
          const uint32_t rowb = v16 + (c >> 2) * kV16Atom + key * 128;
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
          mbar_arrive(bar(kBVFull));
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
    e = cudaFuncSetAttribute(pa_prefill_kernel<BS>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(pa_pf_prep_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
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
