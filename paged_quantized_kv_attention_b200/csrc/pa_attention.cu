// pa_attention.cu -- fused paged quantised-KV GQA attention for sm_100a.
//
// Work items.  A unit is one (sequence, KV head, group of query rows): the rows
// are the (new token, query head of the GQA group) pairs that read the same
// keys.  They are the N side of the tensor-core tiles, keys the M side
// ("swap-AB"), channels the K side.  A sequence with n KV blocks is split into
// ceil(n / T) items of equal size (flash decoding), T chosen by the planner so
// that the items fill the resident CTAs in whole rounds.  Items are numbered
// densely over the sequences with new tokens: the producer warp of every CTA
// computes the per-sequence item counts and their prefix sums once, from the
// device lengths.  The kernel is persistent: CTA i starts with item i and then
// pulls items from an atomic counter in the workspace.
//
// Per CTA, one producer warp and four consumer warps:
//   producer : per item, bulk-copies the query rows and both per-channel scale
//              rows into one of two item slots, then streams the item's KV
//              blocks (block table -> two 3-D TMA boxes per block: the K rows and
//              the V rows of one head) into the consumers' stage rings, straight
//              after the previous item's blocks.  The next item's index and block
//              table entries are fetched while the current ones stream.
//   consumers: per item, the four warps fold the K scale into the queries and
//              encode them as B-operand fragments in shared memory (each warp a
//              quarter of the work); then each warp takes alternate 32-key groups:
//              ldmatrix (K) -> QK on the tensor cores -> online softmax (exp2
//              domain, running maximum raised only when a logit exceeds it by more
//              than 2^8) -> P^T in fp16 -> ldmatrix.trans (V) -> code -> fp16 ->
//              PV MMA; finally the warps' (m, l, O) are merged through shared
//              memory, the V scale applied once, and the result (or a split
//              partial and its log2-sum-exp) stored.  The last split of a unit to
//              finish merges the partials (arrival counter in the workspace).
//
// QK arithmetic.  INT8 and INT4 caches: the folded query q'' = q' 2^(6 - e_q)
// (|q''| < 64) is split into signed int8 digits q'' = d0 + d1 2^-7 + d2 2^-14
// (+ d3 2^-21), each the B operand of an exact mma.sync m16n8k32 s8 x s8 -> s32
// whose A operand is the raw cache byte (INT4: the nibble shifted into the high
// half of a byte, 16 x code).  FP8 caches: codes -> fp16 in registers, q' as an
// fp16 high part plus an fp16 residual.  With at most 4 rows per item, MMA column
// n carries row n / 2, so a thread holds every digit (or both parts) of one row.
// PV arithmetic.  V codes -> fp16 exactly with one byte permute (INT8:
// 1152 + code) or one logic op (INT4: 1032 + code, 1152 + 16 code); the constant
// is removed once at the end using the row sum of P, which a ones-matrix MMA
// accumulates from exactly the fp16 P values the PV MMA consumed.
//
// Sources: the per-channel K scale folded into Q with a power-of-two normaliser
// (INT4 paged-KV page, onnxruntime PR 32515, Code analysis 3); INT8 codes kept
// raw and converted to FP16 in registers right before an m16n8k16 MMA with FP32
// accumulation (INT8-KV tensor-core page, onnxruntime PR 33707, Code analysis
// 1); online softmax, masking and the flash-decoding split with a partials
// buffer (GQA GEMV decode page, onnxruntime PR 29216, Code analysis 1-2); the
// units sized by the exact max_query_len (exact max_query_len page, onnxruntime
// PR 28409, Code analysis 2).
#include <math.h>

#include <atomic>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

constexpr uint32_t kFull = 0xffffffffu;
constexpr uint32_t kOnesH2 = 0x3C003C00u;  // fp16x2 (1, 1)

// NT: 8-column n-tiles per item (rows = 8 NT).  LP: at most 4 rows per item;
// MMA column n carries row n / 2 (QK: the two halves of a digit/part pair;
// PV: the row twice).
template <int KV, int D, int BS, int NT, bool LP>
struct Cfg {
  static_assert(!LP || NT == 1, "row-pair packing uses one n-tile");
  static constexpr bool kInt = (KV != PA_KV_FP8_E4M3);
  static constexpr int kCHS = (KV == PA_KV_INT4) ? D / 2 : D;  // cache bytes per row
  static constexpr int kTile = BS * kCHS;                       // one block, one head
  static constexpr int kStageBytes = 2 * kTile;                 // K + V
  static constexpr int kChunks = kCHS / 16;                     // 16-byte chunks per row
  static constexpr int kSwzMask = (kCHS == 128) ? 7 : (kCHS == 64) ? 3 : 1;
  static constexpr int kMTiles = D / 16;                        // PV m-tiles (output dims)
  static constexpr int kKeyTiles = BS / 16;                     // 16-key tiles per block
  static constexpr int kBPI = (BS == 16) ? 2 : 1;               // blocks per warp iteration
  static constexpr int kTPI = kBPI * kKeyTiles;                 // key tiles per iteration (2)
  static constexpr int kWarps = 4;                              // consumer warps
  static constexpr int kThreads = (kWarps + 1) * 32;            // + one producer warp
  // ring: one sub-ring of kSW stages per consumer warp (fixed ownership), at
  // least two iterations deep, about 64 KB in total
  static constexpr int kSWRaw = 65536 / (kWarps * kStageBytes);
  static constexpr int kSW = kSWRaw < 2 * kBPI ? 2 * kBPI : (kSWRaw > 16 ? 16 : kSWRaw);
  static constexpr int kStages = kWarps * kSW;
  // producer group: whole warp iterations, at most kSW blocks of any warp, <= 32 lanes
  static constexpr int kItPerGroupRaw = (kSW < 8 ? kSW : 8) / kBPI;
  static constexpr int kGroup = kWarps * kBPI * (kItPerGroupRaw < 1 ? 1 : kItPerGroupRaw);
  static constexpr int kRows = LP ? 4 : 8 * NT;
  // QK accumulator sets per n-tile: integer digits (LP: 2 x 2 digits; else 3),
  // FP8 parts (LP: hi|lo in one; else hi, lo)
  static constexpr int kAcc = kInt ? (LP ? 2 : 3) : (LP ? 1 : 2);
  static constexpr int kDigits = LP ? 4 : 3;
  static constexpr int kKSteps = kInt ? D / 32 : D / 16;
  static constexpr int kQWords = kKSteps * kAcc * 2;            // B-fragment words per lane
  static constexpr int kQStride =
      ((kQWords / 4) % 2 == 0 && kQWords < 32) ? kQWords + 4 : kQWords;  // lds.128 banks
  static constexpr int kUnits = D / 4;                          // 4-channel prologue units per row
  static constexpr int kSlices = LP ? 3 : 1;                    // warp-merge buffers
  static constexpr int kMaxSplits = 128;
  // shared memory map (offsets from the 1024-aligned base)
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kQBytes = kRows * D * 2;                 // query rows of one item slot
  static constexpr int kQOff = kRingBytes;                      // 2 slots
  static constexpr int kKsOff = kQOff + 2 * kQBytes;            // k_scale rows, 2 slots
  static constexpr int kVsOff = kKsOff + 2 * D * 4;             // v_scale rows, 2 slots
  static constexpr int kUnionOff = kVsOff + 2 * D * 4;          // fragments | merge slices | weights
  static constexpr int kFragBytes = NT * 32 * kQStride * 4;
  static constexpr int kSliceBytes = kRows * D * 4;
  static constexpr int kWtsBytes = kMaxSplits * kRows * 4;
  static constexpr int kU0 = kFragBytes > kSlices * kSliceBytes ? kFragBytes : kSlices * kSliceBytes;
  static constexpr int kUnionBytes = kU0 > kWtsBytes ? kU0 : kWtsBytes;
  static constexpr int kBarOff = kUnionOff + kUnionBytes;
  static constexpr int kNumBars = 2 * kStages + 4;              // full, empty, item full/empty
  static constexpr int kDescOff = kBarOff + kNumBars * 8;
  static constexpr int kMLOff = kDescOff + 2 * 64;              // merge m, l: [kSlices][2][kRows]
  static constexpr int kCOff = kMLOff + kSlices * 2 * kRows * 4;  // row logit multipliers
  static constexpr int kFlagOff = kCOff + kRows * 4;
  static constexpr int kSmemBytes = kFlagOff + 16;
  static_assert(kChunks % 2 == 0, "ldmatrix.x4 covers two 16-byte chunks");
  static_assert(kTile % ((kSwzMask + 1) * 128) == 0, "tiles keep the swizzle-atom alignment");
  static_assert(kTPI == 2, "two 16-key tiles per warp iteration");
  static_assert(kStages <= 64, "stage count");
  static_assert(kGroup <= 32 && kGroup / (kWarps * kBPI) * kBPI <= kSW, "producer group");
  static_assert(kQWords % 4 == 0 && kQStride % 4 == 0, "fragment rows are lds.128 aligned");
  static_assert(kUnionOff % 16 == 0, "fragment area alignment");
};

// One work item as published by the producer to the consumers (64 bytes).
struct ItemDesc {
  int valid;  // 0: no more work
  int b, kv, rg, split;
  int q0, row0, row_end, past, kmax, kfull;
  int blk_begin, nloc, Lb, nsplit, pad;
};
static_assert(sizeof(ItemDesc) == 64, "descriptor slot size");

// Byte offset inside a tile written by TMA with the matching swizzle mode: the
// 16-byte chunk index (bits 4..6) is XORed with the 128-byte line index.
template <int MASK>
__device__ __forceinline__ uint32_t swz(uint32_t off) {
  return off ^ (((off >> 7) & MASK) << 4);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// One bulk copy (global -> shared) completing on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// First of the two adjacent output dims held by accumulator elements c0 / c2 of
// PV m-tile mt for a thread with group index g.
template <int KV>
__device__ __forceinline__ int out_dim(int mt, int g) {
  if constexpr (KV == PA_KV_INT4) return 32 * (mt >> 1) + 4 * g + 2 * (mt & 1);
  return 16 * mt + 2 * g;
}

// Column offset of dim pair d in a merge slice row (spreads the four row groups
// of a warp over the banks).
__device__ __forceinline__ int slice_col(int d, int sw) { return d ^ (sw << 3); }

// Items of sequence b (0 if it has no new tokens or its lengths are invalid).
template <int BS>
__device__ __forceinline__ int seq_items(const FwdArgs& a, int rows_cta, int q0, int qb, int Lb,
                                         bool& bad) {
  bad = (q0 < 0 || qb < 0 || qb > Lb || q0 + qb > a.total_q ||
         static_cast<long long>(Lb) > static_cast<long long>(a.maxb) * BS);
  if (bad || qb == 0) return 0;
  const int rg = (qb * a.G + rows_cta - 1) / rows_cta;
  if (rg > a.num_row_groups) {
    bad = true;
    return 0;
  }
  int ns, bps;
  split_geometry((Lb + BS - 1) / BS, a.split_target, a.max_splits, &ns, &bps);
  return a.Hk * rg * ns;
}

// Rows, keys and block range of item `local` of sequence b.  Returns false (and
// leaves d.valid = 0) when the item has no keys (a causal row group that ends
// before this split starts).
template <int BS>
__device__ __forceinline__ bool decode_item(const FwdArgs& a, int rows_cta, int b, int local,
                                            int q0, int qb, int Lb, ItemDesc& d) {
  d.valid = 0;
  const int R = qb * a.G;  // rows of (b, kv): row r = token r / G, head kv * G + r % G
  const int rg_n = (R + rows_cta - 1) / rows_cta;
  int ns, bps;
  split_geometry((Lb + BS - 1) / BS, a.split_target, a.max_splits, &ns, &bps);
  d.split = local % ns;
  const int rest = local / ns;
  d.rg = rest % rg_n;
  d.kv = rest / rg_n;
  d.b = b;
  d.row0 = d.rg * rows_cta;
  d.row_end = min(R, d.row0 + rows_cta);
  d.q0 = q0;
  d.Lb = Lb;
  d.past = Lb - qb;
  const int i_first = d.row0 / a.G, i_last = (d.row_end - 1) / a.G;
  d.kmax = a.causal ? d.past + i_last + 1 : Lb;    // keys seen by some row
  d.kfull = a.causal ? d.past + i_first + 1 : Lb;  // keys seen by every row
  const int nblk = (d.kmax + BS - 1) / BS;
  d.nsplit = (nblk + bps - 1) / bps;               // splits of this unit that have keys
  d.blk_begin = d.split * bps;
  if (d.blk_begin >= nblk) return false;
  d.nloc = min(nblk, d.blk_begin + bps) - d.blk_begin;
  d.valid = 1;
  return true;
}

// Blocks of an item with nloc blocks that consumer warp w takes: warp iterations
// it = w, w + 4, ... each cover blocks it * BPI .. it * BPI + BPI - 1.
template <int BPI>
__device__ __forceinline__ int warp_blocks(int nloc, int w) {
  const int full = nloc / (4 * BPI);
  const int rem = nloc - full * 4 * BPI - w * BPI;
  return full * BPI + (rem <= 0 ? 0 : (rem < BPI ? rem : BPI));
}

// ---------------------------------------------------------------------------
// Query fragments.  The 128 consumer threads fold k_scale into the item's query
// rows and write every lane's B-operand words to `frag` (lane-major, kQStride
// words per lane), plus each row's logit multiplier C to `rowc`:
//   integer caches: logit (log2 units) = C 2^-6 sum_d code_d q''_d, q'' digits
//   FP8           : logit = C sum_d code_d (hi_d + lo_d)
// with C = softmax_scale log2(e) 2^(e_kv + e_q).
// Word layout (per n-tile, per lane (g, tig)): word (s * kAcc + i) * 2 + r is
// b-register r of k-step s for accumulator set i.  Channel of byte / half e:
//   INT8: 32 s + 16 r + 4 tig + e     INT4: 32 s + 8 tig + 2 e + r
//   FP8 : 16 s + 4 tig + 2 r + e (e < 2, one fp16 per half)
// These match the channels ldmatrix hands the same thread for the K operand.
template <int KV, int D, int BS, int NT, bool LP>
__device__ __forceinline__ void build_fragments(const FwdArgs& a, const uint8_t* sq,
                                                const float* sks, int nrows, uint32_t* frag,
                                                float* rowc, int tid) {
  using C = Cfg<KV, D, BS, NT, LP>;
  const int lane = tid & 31;
  float ksmax = 0.f;
#pragma unroll
  for (int d = lane; d < D; d += 32) ksmax = fmaxf(ksmax, fabsf(sks[d]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ksmax = fmaxf(ksmax, __shfl_xor_sync(kFull, ksmax, o));
  if (!isfinite(ksmax) && tid == 0) record_error(a.err, PA_DEVERR_BAD_SCALE);
  int e_kv = 0;
  (void)frexpf(ksmax, &e_kv);
  const float f_kv = ldexpf(1.f, -e_kv);
  const __half* q16 = reinterpret_cast<const __half*>(sq);
  const __nv_bfloat16* qbf = reinterpret_cast<const __nv_bfloat16*>(sq);
  constexpr int kU = C::kUnits;  // 32 (D = 128) or 16 lanes per row
  for (int idx = tid; idx < C::kRows * kU; idx += 128) {
    const int row = idx / kU, u = idx % kU;
    const bool valid = row < nrows;
    int s, r, tq, ch0, cstep;
    if constexpr (KV == PA_KV_INT8) {
      s = u >> 3; r = (u >> 2) & 1; tq = u & 3; ch0 = 32 * s + 16 * r + 4 * tq; cstep = 1;
    } else if constexpr (KV == PA_KV_INT4) {
      s = u >> 3; r = (u >> 2) & 1; tq = u & 3; ch0 = 32 * s + 8 * tq + r; cstep = 2;
    } else {
      s = u >> 2; r = 0; tq = u & 3; ch0 = 16 * s + 4 * tq; cstep = 1;
    }
    float w[4];
    float rmax = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int ch = ch0 + e * cstep;
      float x = 0.f;
      if (valid) x = a.q_bf16 ? __bfloat162float(qbf[row * D + ch]) : __half2float(q16[row * D + ch]);
      w[e] = x * (sks[ch] * f_kv);
      rmax = fmaxf(rmax, fabsf(w[e]));
    }
#pragma unroll
    for (int o = kU / 2; o > 0; o >>= 1) rmax = fmaxf(rmax, __shfl_xor_sync(kFull, rmax, o));
    int e_q = 0;
    (void)frexpf(rmax, &e_q);
    if (u == 0) rowc[row] = ldexpf(a.sm_scale_log2, e_kv + e_q);
    const int nt = LP ? 0 : row >> 3;
    uint32_t* fr = frag + nt * 32 * C::kQStride;
    if constexpr (C::kInt) {
      const float f = ldexpf(1.f, 6 - e_q);
      uint32_t wd[C::kDigits];
#pragma unroll
      for (int dg = 0; dg < C::kDigits; ++dg) wd[dg] = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = w[e] * f;  // |v| < 64; each remainder times 128 stays within +-64
#pragma unroll
        for (int dg = 0; dg < C::kDigits; ++dg) {
          const float t = rintf(v);
          wd[dg] |= (static_cast<uint32_t>(static_cast<int>(t)) & 0xFFu) << (8 * e);
          v = (v - t) * 128.f;
        }
      }
      if constexpr (LP) {
        // column n = 2 row + p: set i carries digit 2 i + p
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          uint32_t* fl = fr + ((2 * row + p) * 4 + tq) * C::kQStride;
#pragma unroll
          for (int i = 0; i < 2; ++i) fl[(s * 2 + i) * 2 + r] = wd[2 * i + p];
        }
      } else {
        uint32_t* fl = fr + ((row & 7) * 4 + tq) * C::kQStride;
#pragma unroll
        for (int i = 0; i < 3; ++i) fl[(s * 3 + i) * 2 + r] = wd[i];
      }
    } else {
      const float f = ldexpf(1.f, -e_q);
      float hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float xn = w[e] * f;  // |xn| < 1
        hi[e] = __half2float(__float2half_rn(xn));
        lo[e] = xn - hi[e];
      }
      const uint32_t h01 = pack_f32x2_to_h2(hi[0], hi[1]), h23 = pack_f32x2_to_h2(hi[2], hi[3]);
      const uint32_t l01 = pack_f32x2_to_h2(lo[0], lo[1]), l23 = pack_f32x2_to_h2(lo[2], lo[3]);
      if constexpr (LP) {
        // column n = 2 row + p: part p (0 high, 1 residual)
        uint32_t* f0 = fr + ((2 * row) * 4 + tq) * C::kQStride;
        uint32_t* f1 = fr + ((2 * row + 1) * 4 + tq) * C::kQStride;
        f0[s * 2 + 0] = h01;
        f0[s * 2 + 1] = h23;
        f1[s * 2 + 0] = l01;
        f1[s * 2 + 1] = l23;
      } else {
        uint32_t* fl = fr + ((row & 7) * 4 + tq) * C::kQStride;
        fl[(s * 2 + 0) * 2 + 0] = h01;
        fl[(s * 2 + 0) * 2 + 1] = h23;
        fl[(s * 2 + 1) * 2 + 0] = l01;
        fl[(s * 2 + 1) * 2 + 1] = l23;
      }
    }
  }
}

// Registers: one n-tile fits 3 CTAs per SM (<= 136 per thread); two n-tiles
// keep 2 CTAs per SM (<= 200 per thread).
template <int KV, int D, int BS, int NT, bool LP>
__global__ void __launch_bounds__(Cfg<KV, D, BS, NT, LP>::kThreads) __maxnreg__(NT == 1 ? 128 : 200)
    pa_fwd_kernel(const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap, const FwdArgs a) {
  using C = Cfg<KV, D, BS, NT, LP>;
  // The dynamic window starts at the CTA's shared-memory base (the kernel has no
  // static shared memory), which the 1024-byte swizzle atoms of the TMA tiles
  // need; a misaligned base is reported instead of computing garbage.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if ((smem_u32(smem) & 1023u) != 0u) {
    if (threadIdx.x == 0) record_error(a.err, PA_DEVERR_BAD_LENGTH);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  ItemDesc* descs = reinterpret_cast<ItemDesc*>(smem + C::kDescOff);
  float* sm_ml = reinterpret_cast<float*>(smem + C::kMLOff);
  float* rowc = reinterpret_cast<float*>(smem + C::kCOff);
  int* sm_flag = reinterpret_cast<int*>(smem + C::kFlagOff);
  uint32_t* frag = reinterpret_cast<uint32_t*>(smem + C::kUnionOff);
  float* slices = reinterpret_cast<float*>(smem + C::kUnionOff);
  float* wts = slices;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  constexpr int rows_cta = C::kRows;

  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + C::kStages + s); };
  auto item_full = [&](int sl) { return smem_u32(bars + 2 * C::kStages + sl); };
  auto item_empty = [&](int sl) { return smem_u32(bars + 2 * C::kStages + 2 + sl); };
  auto k_tile = [&](int s) { return smem + s * C::kStageBytes; };
  auto v_tile = [&](int s) { return smem + s * C::kStageBytes + C::kTile; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int sl = 0; sl < 2; ++sl) {
      mbar_init(item_full(sl), 1);
      mbar_init(item_empty(sl), 1);
    }
    mbar_fence_init();
  }
  __syncthreads();

  // ======================================================== producer warp
  if (warp == C::kWarps) {
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
    }
    const uint64_t policy = l2_evict_first_policy();
    // ---- L2 prefetch of what the first items read right after the lengths:
    // the block table, the scale rows and the queries, each CTA a slice.
    auto prefetch_slice = [&](const void* base, size_t bytes) {
      const size_t lines = (bytes + 127) / 128;
      const size_t per = (lines + gridDim.x - 1) / gridDim.x;
      const size_t lo = blockIdx.x * per;
      const size_t hi = lo + per < lines ? lo + per : lines;
      for (size_t l = lo + lane; l < hi; l += 32) {
        const size_t off = l * 128 < bytes ? l * 128 : bytes - 1;
        prefetch_l2(reinterpret_cast<const uint8_t*>(base) + off);
      }
    };
    prefetch_slice(a.block_table, static_cast<size_t>(a.batch) * a.maxb * 4);
    prefetch_slice(a.k_scale, static_cast<size_t>(a.Hk) * D * 4);
    prefetch_slice(a.v_scale, static_cast<size_t>(a.Hk) * D * 4);
    prefetch_slice(a.q, static_cast<size_t>(a.total_q) * a.H * D * 2);
    // ---- dense item numbering: per-sequence item counts and their prefix sums,
    // sequence 32 k + lane in register k (up to 256 sequences); beyond that the
    // numbering is sparse (every sequence gets the largest count; empty items
    // are skipped).
    constexpr int kMaxK = 8;
    const int nk = (a.batch + 31) >> 5;
    const bool dense = nk <= kMaxK;
    int incl[kMaxK], cnt[kMaxK], sq0[kMaxK], sqb[kMaxK], sL[kMaxK];
    int total = 0, per_seq = 0;
    if (dense) {
#pragma unroll
      for (int k = 0; k < kMaxK; ++k) {
        const int b = 32 * k + lane;
        sq0[k] = sqb[k] = sL[k] = 0;
        if (k < nk && b < a.batch) {
          const int c0 = a.cu_seqlens_q[b], c1 = a.cu_seqlens_q[b + 1];
          sq0[k] = c0;
          sqb[k] = c1 - c0;
          sL[k] = a.seqlens_k[b];
        }
      }
      bool bad_any = false;
#pragma unroll
      for (int k = 0; k < kMaxK; ++k) {
        incl[k] = total;
        cnt[k] = 0;
        if (k < nk) {  // warp-uniform
          bool bad = false;
          cnt[k] = (32 * k + lane < a.batch)
                       ? seq_items<BS>(a, rows_cta, sq0[k], sqb[k], sL[k], bad)
                       : 0;
          bad_any |= bad;
          int x = cnt[k];
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, x, o);
            if (lane >= o) x += y;
          }
          incl[k] = total + x;
          total += __shfl_sync(kFull, x, 31);
        }
      }
      if (bad_any) record_error(a.err, PA_DEVERR_BAD_LENGTH);
    } else {
      const int max_rg = a.num_row_groups;
      per_seq = a.Hk * max_rg * a.max_splits;
      total = a.batch * per_seq;
    }

    // Item w -> (sequence, index within the sequence, its lengths); false when
    // the item has no work.
    auto locate = [&](int w, ItemDesc& d) -> bool {
      d.valid = 0;
      if (dense) {
#pragma unroll
        for (int k = 0; k < kMaxK; ++k) {
          if (k >= nk) break;
          const unsigned m = __ballot_sync(kFull, incl[k] > w);
          if (m != 0u) {
            const int l = __ffs(m) - 1;
            const int base = __shfl_sync(kFull, incl[k] - cnt[k], l);
            const int q0 = __shfl_sync(kFull, sq0[k], l);
            const int qb = __shfl_sync(kFull, sqb[k], l);
            const int Lb = __shfl_sync(kFull, sL[k], l);
            return decode_item<BS>(a, rows_cta, 32 * k + l, w - base, q0, qb, Lb, d);
          }
        }
        return false;
      }
      const int b = w / per_seq;
      int v = 0;
      if (lane == 0) v = a.cu_seqlens_q[b];
      else if (lane == 1) v = a.cu_seqlens_q[b + 1];
      else if (lane == 2) v = a.seqlens_k[b];
      const int q0 = __shfl_sync(kFull, v, 0);
      const int qb = __shfl_sync(kFull, v, 1) - q0;
      const int Lb = __shfl_sync(kFull, v, 2);
      bool bad = false;
      if (seq_items<BS>(a, rows_cta, q0, qb, Lb, bad) == 0) {
        if (bad) record_error(a.err, PA_DEVERR_BAD_LENGTH);
        return false;
      }
      int local = w - b * per_seq;
      // sparse layout: split fastest over max_splits, then row group, then head
      const int split = local % a.max_splits;
      const int rest = local / a.max_splits;
      const int rg = rest % a.num_row_groups, kv = rest / a.num_row_groups;
      const int R = qb * a.G;
      const int rg_n = (R + rows_cta - 1) / rows_cta;
      int ns, bps;
      split_geometry((Lb + BS - 1) / BS, a.split_target, a.max_splits, &ns, &bps);
      if (rg >= rg_n || split >= ns) return false;
      return decode_item<BS>(a, rows_cta, b, (kv * rg_n + rg) * ns + split, q0, qb, Lb, d);
    };

    int uses[2] = {0, 0};
    int slot = 0;
    // Blocks handed to each consumer warp so far: warp w's k-th block lives in
    // stage w * kSW + k % kSW of its own sub-ring, round k / kSW.
    int cnt_w0 = 0, cnt_w1 = 0, cnt_w2 = 0, cnt_w3 = 0;
    auto cnt_of = [&](int wq) {
      return wq == 0 ? cnt_w0 : (wq == 1 ? cnt_w1 : (wq == 2 ? cnt_w2 : cnt_w3));
    };
    bool ok = true;
    int w = blockIdx.x;  // first item without an atomic
    uint32_t w_pref = 0;
    if (lane == 0) w_pref = atomicAdd(a.work, 1u);  // next index, in flight
    auto next_index = [&]() {
      const int nxt = static_cast<int>(gridDim.x + __shfl_sync(kFull, w_pref, 0));
      if (lane == 0) w_pref = atomicAdd(a.work, 1u);
      return nxt;
    };
    while (ok) {
      ItemDesc d = {};
      while (w < total) {
        if (locate(w, d)) break;
        w = next_index();
      }
      // block-table entries of the item's first group, fetched with the publish
      const int32_t* bt = a.block_table + static_cast<size_t>(d.b) * a.maxb + d.blk_begin;
      int phys_cur = 0;
      if (d.valid && lane < C::kGroup && lane < d.nloc) phys_cur = __ldg(bt + lane);
      // publish the item (or the end marker) in the next slot
      if (lane == 0) {
        if (uses[slot] > 0 && !mbar_wait(item_empty(slot), (uses[slot] - 1) & 1)) {
          record_error(a.err, PA_DEVERR_TIMEOUT);
          ok = false;
        } else {
          descs[slot] = d;
          if (d.valid) {
            const uint32_t row_bytes = D * 2;
            const uint32_t tot =
                static_cast<uint32_t>(d.row_end - d.row0) * row_bytes + 2 * D * 4;
            mbar_arrive_expect_tx(item_full(slot), tot);
            const int i_first = d.row0 / a.G, i_last = (d.row_end - 1) / a.G;
            for (int i = i_first; i <= i_last; ++i) {
              const int r_lo = max(d.row0, i * a.G), r_hi = min(d.row_end, (i + 1) * a.G);
              const uint8_t* src = reinterpret_cast<const uint8_t*>(a.q) +
                                   ((static_cast<size_t>(d.q0 + i) * a.H + d.kv * a.G +
                                     (r_lo - i * a.G)) * D) * 2;
              bulk_load(smem_u32(smem + C::kQOff + slot * C::kQBytes + (r_lo - d.row0) * row_bytes),
                        src, static_cast<uint32_t>(r_hi - r_lo) * row_bytes, item_full(slot));
            }
            bulk_load(smem_u32(smem + C::kKsOff + slot * D * 4), a.k_scale + d.kv * D, D * 4,
                      item_full(slot));
            bulk_load(smem_u32(smem + C::kVsOff + slot * D * 4), a.v_scale + d.kv * D, D * 4,
                      item_full(slot));
          } else {
            mbar_arrive(item_full(slot));
          }
        }
      }
      ok = __shfl_sync(kFull, ok, 0);
      ++uses[slot];
      if (!ok || !d.valid) break;

      // Blocks go out in groups of kGroup (whole warp iterations, at most kSW
      // blocks of any warp, so every block of a group has its own stage): lane j
      // waits for its stage to be released, arms it and issues the two boxes, all
      // lanes in parallel; the next group's block-table entries are loaded first.
      // Item block lb belongs to warp (lb / kBPI) % 4, the split the consumers use.
      constexpr int kGroup = C::kGroup;
      for (int base = 0; base < d.nloc && ok; base += kGroup) {
        const int lb = base + lane;
        int phys_nxt = 0;
        if (lane < kGroup && lb + kGroup < d.nloc) phys_nxt = __ldg(bt + lb + kGroup);
        bool mine_ok = true;
        if (lane < kGroup && lb < d.nloc) {
          int phys = phys_cur;
          if (phys < 0 || phys >= a.num_blocks) {
            record_error(a.err, PA_DEVERR_BAD_BLOCK);
            phys = a.num_blocks;  // out-of-range box: TMA fills zeros, nothing faults
          }
          const int wq = (lb / C::kBPI) % C::kWarps;
          const int k = cnt_of(wq) + (lb / (C::kWarps * C::kBPI)) * C::kBPI + lb % C::kBPI;
          const int s = wq * C::kSW + k % C::kSW;
          const int round = k / C::kSW;
          if (round > 0 && !mbar_wait(empty_bar(s), (round - 1) & 1)) {
            mine_ok = false;
          } else {
            mbar_arrive_expect_tx(full_bar(s), C::kStageBytes);
            tma_load_3d(smem_u32(k_tile(s)), &kmap, full_bar(s), 0, d.kv, phys * BS, policy);
            tma_load_3d(smem_u32(v_tile(s)), &vmap, full_bar(s), 0, d.kv, phys * BS, policy);
          }
        }
        phys_cur = phys_nxt;
        ok = __all_sync(kFull, mine_ok);
        if (!ok && lane == 0) record_error(a.err, PA_DEVERR_TIMEOUT);
      }
      cnt_w0 += warp_blocks<C::kBPI>(d.nloc, 0);
      cnt_w1 += warp_blocks<C::kBPI>(d.nloc, 1);
      cnt_w2 += warp_blocks<C::kBPI>(d.nloc, 2);
      cnt_w3 += warp_blocks<C::kBPI>(d.nloc, 3);
      slot ^= 1;
      w = next_index();
    }
    // The last prefetched index is consumed (its atomic has completed) before
    // this CTA signs off.
    const uint32_t last = __shfl_sync(kFull, w_pref, 0);
    // Leave no copy in flight: wait for the last box of every stage, all within
    // one bounded window (the consumers normally consumed them already).
    if (lane == 0) {
      const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
      bool fine = true;
      for (int wq = 0; wq < C::kWarps; ++wq)
        for (int j = 0; fine && j < C::kSW && j < cnt_of(wq); ++j) {
          const int last_round = (cnt_of(wq) - 1 - j) / C::kSW;
          fine = mbar_wait_until(full_bar(wq * C::kSW + j), last_round & 1, deadline);
        }
      if (!fine) record_error(a.err, PA_DEVERR_TIMEOUT);
      __threadfence();
      // The last CTA to finish rewinds the work counter for the next call.
      if (last == 0xffffffffu) record_error(a.err, PA_DEVERR_BAD_LENGTH);  // (never: uses the value)
      if (atomicAdd(a.work + 1, 1u) == gridDim.x - 1) {
        a.work[0] = 0u;
        a.work[1] = 0u;
      }
    }
    return;
  }

  // ======================================================== consumer warps
  const int tid = threadIdx.x;  // 0..127
  int uses[2] = {0, 0};
  int slot = 0;
  int kc = 0;  // blocks this warp consumed so far: its k-th block is in stage
               // warp * kSW + k % kSW of its own sub-ring, round k / kSW
  // ldmatrix lane addressing: matrix (lane >> 3) covers rows (lane & 7) + 8 * (m & 1)
  // of a 16-row key tile and chunk (2 cp + (m >> 1)).
  const int lm = lane >> 3;
  const int ld_row = (lane & 7) + 8 * (lm & 1);
  const int ld_chunk = lm >> 1;

  for (;;) {
    if (!mbar_wait(item_full(slot), uses[slot] & 1)) {
      if (lane == 0) record_error(a.err, PA_DEVERR_TIMEOUT);
      break;
    }
    ++uses[slot];
    const ItemDesc d = descs[slot];
    if (!d.valid) break;
    const int kv = d.kv, rg = d.rg, b = d.b, split = d.split, q0 = d.q0;
    const int row0 = d.row0, row_end = d.row_end, past = d.past, kmax = d.kmax, kfull = d.kfull;
    const int blk_begin = d.blk_begin, nloc = d.nloc, nsplit = d.nsplit;
    const int Lb = d.Lb;
    const int nrows = row_end - row0;
    const float* sks = reinterpret_cast<const float*>(smem + C::kKsOff) + slot * D;
    const float* svs = reinterpret_cast<const float*>(smem + C::kVsOff) + slot * D;
    bool alive = true;

    // ---- prologue: query fragments for this item (cooperative)
    build_fragments<KV, D, BS, NT, LP>(a, smem + C::kQOff + slot * C::kQBytes, sks, nrows, frag,
                                       rowc, tid);
    consumer_sync();
    uint32_t qf[NT][C::kQWords];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int k4 = 0; k4 < C::kQWords / 4; ++k4) {
        const uint4 v = *reinterpret_cast<const uint4*>(
            frag + (nt * 32 + lane) * C::kQStride + 4 * k4);
        qf[nt][4 * k4 + 0] = v.x;
        qf[nt][4 * k4 + 1] = v.y;
        qf[nt][4 * k4 + 2] = v.z;
        qf[nt][4 * k4 + 3] = v.w;
      }
    // per accumulator column j: logit weights and causal limit (LP: j = 0 only,
    // the thread's row is tig)
    float wA[NT][2], wB[NT][2];
    int lim[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int rl = LP ? tig : nt * 8 + 2 * tig + j;
        const float cr = rowc[rl];
        if constexpr (C::kInt) {
          const float base = cr * ((KV == PA_KV_INT4) ? (1.f / 131072.f) : (1.f / 8192.f));
          wA[nt][j] = base;                                            // C 2^-13 (/16 INT4)
          wB[nt][j] = LP ? base * (1.f / 16384.f) : base * (1.f / 128.f);  // digits 2|3 or 2
        } else {
          wA[nt][j] = cr;
          wB[nt][j] = 0.f;
        }
        lim[nt][j] = (row0 + rl < row_end && a.causal) ? past + (row0 + rl) / a.G : kmax - 1;
      }
    consumer_sync();  // every warp holds its fragments: the area may be reused

    float o[NT][C::kMTiles][4];
    float lacc[NT][4];  // row sums of the fp16 P (ones-matrix MMA)
    float m_run[NT][2], msub[NT][2], thr[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int mt = 0; mt < C::kMTiles; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[nt][mt][e] = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) lacc[nt][e] = 0.f;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        m_run[nt][j] = -INFINITY;
        msub[nt][j] = 0.f;
        thr[nt][j] = -INFINITY;
      }
    }

    for (int it = warp; alive && it * C::kBPI < nloc; it += C::kWarps) {
      const int lb0 = it * C::kBPI;
      const int nb = min(C::kBPI, nloc - lb0);
      const int ntiles = nb * C::kKeyTiles;
      for (int bi = 0; bi < nb; ++bi) {
        // The stage is this warp's own: it consumed round - 1 itself, so the
        // parity of the wait is unambiguous.
        const int k = kc + bi;
        const int s = warp * C::kSW + k % C::kSW, round = k / C::kSW;
        if (!mbar_wait(full_bar(s), round & 1)) {
          if (lane == 0) record_error(a.err, PA_DEVERR_TIMEOUT);
          alive = false;
        }
      }
      if (!alive) break;

      // X: logits in log2 units minus the row's running reference, then P.
      // LP: X[t][0][eh] = key g + 8 eh of row tig.  Else X[t][nt][e]: key g + 8 (e >> 1),
      // row nt * 8 + 2 tig + (e & 1).
      float X[C::kTPI][NT][4];
#pragma unroll
      for (int t = 0; t < C::kTPI; ++t) {
        if (t >= ntiles) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) X[t][nt][e] = -INFINITY;
          continue;
        }
        const int bi = t / C::kKeyTiles, kt = t % C::kKeyTiles;
        const uint32_t kbase = smem_u32(k_tile(warp * C::kSW + (kc + bi) % C::kSW));
        const int key0 = (blk_begin + lb0 + bi) * BS + kt * 16;
        const bool need_mask = key0 + 16 > kfull;
        if constexpr (C::kInt) {
          int acc[C::kAcc][NT][4];
#pragma unroll
          for (int i = 0; i < C::kAcc; ++i)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[i][nt][e] = 0;
#pragma unroll
          for (int cp = 0; cp < C::kChunks / 2; ++cp) {
            uint32_t r[4];
            const uint32_t off = (kt * 16 + ld_row) * C::kCHS + (2 * cp + ld_chunk) * 16;
            ldsm_x4(kbase + swz<C::kSwzMask>(off), r);
#pragma unroll
            for (int h = 0; h < (KV == PA_KV_INT4 ? 2 : 1); ++h) {
              uint32_t a0, a1, a2, a3;
              int s;
              if constexpr (KV == PA_KV_INT8) {
                a0 = r[0]; a1 = r[1]; a2 = r[2]; a3 = r[3];  // 32 channels, raw codes
                s = cp;
              } else {
                // nibbles as signed bytes 16 x code: low nibbles shifted up, high masked
                const uint32_t x0 = r[2 * h], x1 = r[2 * h + 1];  // keys g, g+8; chunk 2cp+h
                a0 = (x0 << 4) & 0xF0F0F0F0u;
                a1 = (x1 << 4) & 0xF0F0F0F0u;
                a2 = x0 & 0xF0F0F0F0u;
                a3 = x1 & 0xF0F0F0F0u;
                s = 2 * cp + h;
              }
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < C::kAcc; ++i)
                  imma_16832<false>(acc[i][nt], a0, a1, a2, a3, qf[nt][(s * C::kAcc + i) * 2],
                                    qf[nt][(s * C::kAcc + i) * 2 + 1]);
            }
          }
          if constexpr (LP) {
#pragma unroll
            for (int eh = 0; eh < 2; ++eh) {
              const int A = acc[0][0][2 * eh] * 128 + acc[0][0][2 * eh + 1];
              const int B2 = acc[1][0][2 * eh] * 128 + acc[1][0][2 * eh + 1];
              float xv = fmaf(__int2float_rn(A), wA[0][0],
                              fmaf(__int2float_rn(B2), wB[0][0], -msub[0][0]));
              if (need_mask && key0 + g + 8 * eh > lim[0][0]) xv = -INFINITY;
              X[t][0][eh] = xv;
            }
          } else {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = e & 1;
                const int A = acc[0][nt][e] * 128 + acc[1][nt][e];
                float xv = fmaf(__int2float_rn(A), wA[nt][j],
                                fmaf(__int2float_rn(acc[2][nt][e]), wB[nt][j], -msub[nt][j]));
                if (need_mask && key0 + g + (e >> 1) * 8 > lim[nt][j]) xv = -INFINITY;
                X[t][nt][e] = xv;
              }
          }
        } else {
          float sacc[C::kAcc][NT][4];
#pragma unroll
          for (int i = 0; i < C::kAcc; ++i)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) sacc[i][nt][e] = 0.f;
#pragma unroll
          for (int cp = 0; cp < C::kChunks / 2; ++cp) {
            uint32_t r[4];
            const uint32_t off = (kt * 16 + ld_row) * C::kCHS + (2 * cp + ld_chunk) * 16;
            ldsm_x4(kbase + swz<C::kSwzMask>(off), r);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int s = 2 * cp + h;  // 16-channel k-step
              uint32_t a0, a1, a2, a3;
              e4m3x4_to_h2x2(r[2 * h], a0, a2);      // key g: channels +0,1 | +2,3
              e4m3x4_to_h2x2(r[2 * h + 1], a1, a3);  // key g+8
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < C::kAcc; ++i)
                  mma_16816(sacc[i][nt], a0, a1, a2, a3, qf[nt][(s * C::kAcc + i) * 2],
                            qf[nt][(s * C::kAcc + i) * 2 + 1]);
            }
          }
          if constexpr (LP) {
#pragma unroll
            for (int eh = 0; eh < 2; ++eh) {
              // columns 2 tig / 2 tig + 1: high part / residual of row tig
              float xv = fmaf(sacc[0][0][2 * eh] + sacc[0][0][2 * eh + 1], wA[0][0], -msub[0][0]);
              if (need_mask && key0 + g + 8 * eh > lim[0][0]) xv = -INFINITY;
              X[t][0][eh] = xv;
            }
          } else {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = e & 1;
                float xv = fmaf(sacc[0][nt][e] + sacc[1][nt][e], wA[nt][j], -msub[nt][j]);
                if (need_mask && key0 + g + (e >> 1) * 8 > lim[nt][j]) xv = -INFINITY;
                X[t][nt][e] = xv;
              }
          }
        }
      }

      // ---------------- online softmax with a lazily raised running max
      if constexpr (LP) {
        float mx = fmaxf(fmaxf(X[0][0][0], X[0][0][1]), fmaxf(X[1][0][0], X[1][0][1]));
        if (__any_sync(kFull, mx > thr[0][0])) {
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
          if (mx > thr[0][0]) {
            const float mnew = mx + msub[0][0];
            const float alpha = (m_run[0][0] == -INFINITY) ? 0.f : fast_exp2(m_run[0][0] - mnew);
#pragma unroll
            for (int mt = 0; mt < C::kMTiles; ++mt)
#pragma unroll
              for (int e = 0; e < 4; ++e) o[0][mt][e] *= alpha;
#pragma unroll
            for (int e = 0; e < 4; ++e) lacc[0][e] *= alpha;
#pragma unroll
            for (int t = 0; t < C::kTPI; ++t) {
              X[t][0][0] -= mx;
              X[t][0][1] -= mx;
            }
            m_run[0][0] = mnew;
            msub[0][0] = mnew;
            thr[0][0] = 8.f;
          }
        }
#pragma unroll
        for (int t = 0; t < C::kTPI; ++t) {
          X[t][0][0] = fast_exp2(X[t][0][0]);  // <= 2^8: safe range for fp16
          X[t][0][1] = fast_exp2(X[t][0][1]);
        }
      } else {
        float mx[NT][2];
        bool any = false;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            mx[nt][j] = fmaxf(fmaxf(X[0][nt][j], X[0][nt][j + 2]),
                              fmaxf(X[1][nt][j], X[1][nt][j + 2]));
            any |= mx[nt][j] > thr[nt][j];
          }
        if (__any_sync(kFull, any)) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              float m = mx[nt][j];
              m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
              m = fmaxf(m, __shfl_xor_sync(kFull, m, 8));
              m = fmaxf(m, __shfl_xor_sync(kFull, m, 16));
              if (m > thr[nt][j]) {
                const float mnew = m + msub[nt][j];
                const float alpha =
                    (m_run[nt][j] == -INFINITY) ? 0.f : fast_exp2(m_run[nt][j] - mnew);
#pragma unroll
                for (int mt = 0; mt < C::kMTiles; ++mt) {
                  o[nt][mt][j] *= alpha;
                  o[nt][mt][j + 2] *= alpha;
                }
                lacc[nt][j] *= alpha;
                lacc[nt][j + 2] *= alpha;
#pragma unroll
                for (int t = 0; t < C::kTPI; ++t) {
                  X[t][nt][j] -= m;
                  X[t][nt][j + 2] -= m;
                }
                m_run[nt][j] = mnew;
                msub[nt][j] = mnew;
                thr[nt][j] = 8.f;
              }
            }
        }
#pragma unroll
        for (int t = 0; t < C::kTPI; ++t)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) X[t][nt][e] = fast_exp2(X[t][nt][e]);
      }

      // ---------------- O^T[dim, col] += V^T P^T, per key tile
#pragma unroll
      for (int t = 0; t < C::kTPI; ++t) {
        if (t >= ntiles) continue;
        const int bi = t / C::kKeyTiles, kt = t % C::kKeyTiles;
        const uint32_t vbase = smem_u32(v_tile(warp * C::kSW + (kc + bi) % C::kSW));
        uint32_t pb[NT][2];
        if constexpr (LP) {
          // (row tig; keys g, g+8) -> column n = g: b0 (keys 2tig, 2tig+1) and b1
          // (keys 2tig+8, 2tig+9) of row n / 2; movmatrix gives even lanes b0 and
          // odd lanes b1, the partner lane (lane ^ 4) the other.
          const uint32_t p = pack_f32x2_to_h2(X[t][0][0], X[t][0][1]);
          const uint32_t mtr = movmatrix_trans(p);
          const uint32_t y = __shfl_xor_sync(kFull, mtr, 4);
          pb[0][0] = (g & 1) ? y : mtr;
          pb[0][1] = (g & 1) ? mtr : y;
        } else {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            pb[nt][0] = movmatrix_trans(pack_f32x2_to_h2(X[t][nt][0], X[t][nt][1]));
            pb[nt][1] = movmatrix_trans(pack_f32x2_to_h2(X[t][nt][2], X[t][nt][3]));
          }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_16816(lacc[nt], kOnesH2, kOnesH2, kOnesH2, kOnesH2, pb[nt][0], pb[nt][1]);
        const int tkey0 = (blk_begin + lb0 + bi) * BS + kt * 16;
#pragma unroll
        for (int cp = 0; cp < C::kChunks / 2; ++cp) {
          uint32_t r[4];
          const uint32_t off = (kt * 16 + ld_row) * C::kCHS + (2 * cp + ld_chunk) * 16;
          ldsm_x4_trans(vbase + swz<C::kSwzMask>(off), r);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t lo = r[2 * h], hi = r[2 * h + 1];  // keys 2tig.. / 2tig+8.. of chunk c
            const int c = 2 * cp + h;
#pragma unroll
            for (int hh = 0; hh < (KV == PA_KV_INT4 ? 2 : 1); ++hh) {
              uint32_t a0, a1, a2, a3;
              int mt;
              if constexpr (KV == PA_KV_INT8) {
                // fp16 1024 + (code + 128) = 1152 + code
                const uint32_t ylo = lo ^ 0x80808080u, yhi = hi ^ 0x80808080u;
                a0 = prmt(ylo, 0x64646464u, 0x4240);
                a1 = prmt(ylo, 0x64646464u, 0x4341);
                a2 = prmt(yhi, 0x64646464u, 0x4240);
                a3 = prmt(yhi, 0x64646464u, 0x4341);
                mt = c;
              } else if constexpr (KV == PA_KV_FP8_E4M3) {
                e4m3x4_to_h2x2(prmt(lo, 0u, 0x3120), a0, a1);
                e4m3x4_to_h2x2(prmt(hi, 0u, 0x3120), a2, a3);
                if (tkey0 + 16 > Lb) {
                  // Keys past the sequence end hold stale bytes; an FP8 NaN there would
                  // poison P*V even with P = 0, so such V codes are zeroed.
                  const int kb = tkey0 + 2 * tig;
                  const uint32_t mlo = (kb < Lb ? 0x0000ffffu : 0u) | (kb + 1 < Lb ? 0xffff0000u : 0u);
                  const uint32_t mhi =
                      (kb + 8 < Lb ? 0x0000ffffu : 0u) | (kb + 9 < Lb ? 0xffff0000u : 0u);
                  a0 &= mlo;
                  a1 &= mlo;
                  a2 &= mhi;
                  a3 &= mhi;
                }
                mt = c;
              } else {
                // low nibble: fp16 1024 + (code + 8); high nibble: 1024 + 16 (code + 8)
                const uint32_t zl = hh ? (lo >> 8) : lo, zh = hh ? (hi >> 8) : hi;
                a0 = (zl & 0x000F000Fu) ^ 0x64086408u;
                a1 = (zl & 0x00F000F0u) ^ 0x64806480u;
                a2 = (zh & 0x000F000Fu) ^ 0x64086408u;
                a3 = (zh & 0x00F000F0u) ^ 0x64806480u;
                mt = 2 * c + hh;
              }
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                mma_16816(o[nt][mt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0)
        for (int bi = 0; bi < nb; ++bi) mbar_arrive(empty_bar(warp * C::kSW + (kc + bi) % C::kSW));
      kc += nb;
    }

    // ---- this warp's result: remove the code->fp16 constants (using the exact
    // row sums of P); columns j of the accumulators (LP: both = row tig)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int mt = 0; mt < C::kMTiles; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float l = lacc[nt][LP ? 0 : (e & 1)];
          if constexpr (KV == PA_KV_INT8) {
            o[nt][mt][e] = fmaf(-1152.f, l, o[nt][mt][e]);
          } else if constexpr (KV == PA_KV_INT4) {
            o[nt][mt][e] = (e < 2) ? fmaf(-1032.f, l, o[nt][mt][e])
                                   : fmaf(-1152.f, l, o[nt][mt][e]) * (1.f / 16.f);
          }
        }

    // ---- merge the four warps' (m, l, O); warp 0 ends with the total.
    // Slice rows are [row][D] fp32 with swizzled dim pairs.
    auto slice_sw = [&](int row) { return LP ? (row & 3) : ((row >> 1) & 3); };
    auto write_slice = [&](float* sl, float* ml) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < (LP ? 1 : 2); ++j) {
          const int row = LP ? tig : nt * 8 + 2 * tig + j;
#pragma unroll
          for (int mt = 0; mt < C::kMTiles; ++mt) {
            const int dcol = slice_col(out_dim<KV>(mt, g), slice_sw(row));
            *reinterpret_cast<float2*>(sl + row * D + dcol) =
                make_float2(o[nt][mt][j], o[nt][mt][j + 2]);
          }
          if (g == 0) {
            ml[row] = m_run[nt][j];
            ml[C::kRows + row] = lacc[nt][LP ? 0 : j];
          }
        }
    };
    // Adds a slice (m_s, l_s, O_s) into this warp's (m, l, O).
    auto merge_slice = [&](const float* sl, const float* ml) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < (LP ? 1 : 2); ++j) {
          const int row = LP ? tig : nt * 8 + 2 * tig + j;
          const float ms = ml[row], ls = ml[C::kRows + row];
          const float M = fmaxf(m_run[nt][j], ms);
          const float fo = (m_run[nt][j] == -INFINITY) ? 0.f : fast_exp2(m_run[nt][j] - M);
          const float fs = (ms == -INFINITY) ? 0.f : fast_exp2(ms - M);
#pragma unroll
          for (int mt = 0; mt < C::kMTiles; ++mt) {
            const int dcol = slice_col(out_dim<KV>(mt, g), slice_sw(row));
            const float2 v = *reinterpret_cast<const float2*>(sl + row * D + dcol);
            o[nt][mt][j] = fmaf(v.x, fs, o[nt][mt][j] * fo);
            o[nt][mt][j + 2] = fmaf(v.y, fs, o[nt][mt][j + 2] * fo);
          }
          const int jl = LP ? 0 : j;
          lacc[nt][jl] = fmaf(ls, fs, lacc[nt][jl] * fo);
          m_run[nt][j] = M;
        }
    };
    if constexpr (LP) {
      if (warp > 0) write_slice(slices + (warp - 1) * C::kSliceBytes / 4,
                                sm_ml + (warp - 1) * 2 * C::kRows);
      consumer_sync();
      if (warp == 0)
#pragma unroll
        for (int sl = 0; sl < C::kSlices; ++sl)
          merge_slice(slices + sl * C::kSliceBytes / 4, sm_ml + sl * 2 * C::kRows);
      consumer_sync();
    } else {
      for (int wsum = C::kWarps - 1; wsum >= 0; --wsum) {
        if (warp == wsum) {
          if (wsum != C::kWarps - 1) merge_slice(slices, sm_ml);
          if (wsum != 0) write_slice(slices, sm_ml);
        }
        consumer_sync();
      }
    }

    // ---- warp 0: normalise, apply the V scale, store the output or the split partial
    if (warp == 0) {
      const bool is_split = nsplit > 1;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < (LP ? 1 : 2); ++j) {
          const int rl = LP ? tig : nt * 8 + 2 * tig + j;
          if (rl >= nrows) continue;
          const int r = row0 + rl;
          const size_t orow = static_cast<size_t>(q0 + r / a.G) * a.H + kv * a.G + r % a.G;
          const float L = lacc[nt][LP ? 0 : j];
          const float inv = (L > 0.f) ? 1.f / L : 0.f;
          const size_t prow = static_cast<size_t>(split) * a.total_q * a.H + orow;
#pragma unroll
          for (int mt = 0; mt < C::kMTiles; ++mt) {
            const int dd = out_dim<KV>(mt, g);
            const float2 vs = *reinterpret_cast<const float2*>(svs + dd);
            const float o0 = o[nt][mt][j] * inv * vs.x;
            const float o1 = o[nt][mt][j + 2] * inv * vs.y;
            if (!is_split) {
              if (a.out_bf16)
                *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(a.out) +
                                                   orow * D + dd) = __floats2bfloat162_rn(o0, o1);
              else
                *reinterpret_cast<__half2*>(reinterpret_cast<__half*>(a.out) + orow * D + dd) =
                    __floats2half2_rn(o0, o1);
            } else {
              *reinterpret_cast<float2*>(a.o_part + prow * D + dd) = make_float2(o0, o1);
            }
          }
          if (is_split && g == 0)
            a.lse_part[prow] = (L > 0.f) ? m_run[nt][j] + __log2f(L) : -INFINITY;
        }
      if (is_split) {
        // publish this split and count arrivals; the last split of the unit
        // merges all of them and rewinds the counter for the next call
        __threadfence();
        __syncwarp();
        uint32_t* counter =
            a.counters + (static_cast<size_t>(b) * a.Hk + kv) * a.num_row_groups + rg;
        int last = 0;
        if (lane == 0) last = (atomicAdd(counter, 1u) == static_cast<uint32_t>(nsplit - 1));
        last = __shfl_sync(kFull, last, 0);
        if (lane == 0) *sm_flag = last;
      }
      if (lane == 0 && !is_split) *sm_flag = 0;
    }
    if (nsplit > 1) {
      consumer_sync();
      if (*sm_flag) {
        __threadfence();
        const size_t stride = static_cast<size_t>(a.total_q) * a.H;
        const int S = nsplit;
        const int nthr = C::kWarps * 32;
        // 1) every (split, row) log2-sum-exp
        for (int idx = tid; idx < S * nrows; idx += nthr) {
          const int s = idx / nrows, row = idx % nrows;
          const int r = row0 + row;
          const size_t orow = static_cast<size_t>(q0 + r / a.G) * a.H + kv * a.G + r % a.G;
          wts[s * C::kRows + row] = __ldcg(a.lse_part + s * stride + orow);
        }
        consumer_sync();
        // 2) per row (one warp per row): weights 2^(lse_s - max) / sum
        for (int row = warp; row < nrows; row += C::kWarps) {
          float M = -INFINITY;
          for (int s = lane; s < S; s += 32) M = fmaxf(M, wts[s * C::kRows + row]);
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o2));
          float sum = 0.f;
          for (int s = lane; s < S; s += 32) {
            const float ls = wts[s * C::kRows + row];
            const float wgt = (ls == -INFINITY) ? 0.f : fast_exp2(ls - M);
            wts[s * C::kRows + row] = wgt;
            sum += wgt;
          }
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 >>= 1) sum += __shfl_xor_sync(kFull, sum, o2);
          const float inv = sum > 0.f ? 1.f / sum : 0.f;
          __syncwarp();
          for (int s = lane; s < S; s += 32) wts[s * C::kRows + row] *= inv;
        }
        consumer_sync();
        // 3) weighted sum of the partials, eight splits in flight per thread
        for (int idx = tid; idx < nrows * (D / 4); idx += nthr) {
          const int row = idx / (D / 4);
          const int dd = (idx % (D / 4)) * 4;
          const int r = row0 + row;
          const size_t orow = static_cast<size_t>(q0 + r / a.G) * a.H + kv * a.G + r % a.G;
          const float* base = a.o_part + orow * D + dd;
          float4 acc4 = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int s8 = 0; s8 < S; s8 += 8) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
              v[u] = (s8 + u < S)
                         ? __ldcg(reinterpret_cast<const float4*>(base + (s8 + u) * stride * D))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              if (s8 + u < S) {
                const float wgt = wts[(s8 + u) * C::kRows + row];
                acc4.x = fmaf(wgt, v[u].x, acc4.x);
                acc4.y = fmaf(wgt, v[u].y, acc4.y);
                acc4.z = fmaf(wgt, v[u].z, acc4.z);
                acc4.w = fmaf(wgt, v[u].w, acc4.w);
              }
            }
          }
          if (a.out_bf16) {
            __nv_bfloat162* dst =
                reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(a.out) +
                                                  orow * D + dd);
            dst[0] = __floats2bfloat162_rn(acc4.x, acc4.y);
            dst[1] = __floats2bfloat162_rn(acc4.z, acc4.w);
          } else {
            __half2* dst = reinterpret_cast<__half2*>(reinterpret_cast<__half*>(a.out) + orow * D + dd);
            dst[0] = __floats2half2_rn(acc4.x, acc4.y);
            dst[1] = __floats2half2_rn(acc4.z, acc4.w);
          }
        }
        if (tid == 0)
          a.counters[(static_cast<size_t>(b) * a.Hk + kv) * a.num_row_groups + rg] = 0u;
      }
      consumer_sync();  // weights / flag consumed before the next item's prologue
    }
    // the item slot (query rows, scales, descriptor) may be refilled
    if (warp == 0) {
      __syncwarp();
      if (lane == 0) mbar_arrive(item_empty(slot));
    }
    slot ^= 1;
  }
}

template <int KV, int D, int BS, int NT, bool LP>
static cudaError_t launch_t(const CUtensorMap& kmap, const CUtensorMap& vmap, FwdArgs a,
                            cudaStream_t stream) {
  using C = Cfg<KV, D, BS, NT, LP>;
  auto kern = pa_fwd_kernel<KV, D, BS, NT, LP>;
  // Per device: the dynamic shared-memory opt-in and the resident CTAs per SM.
  static std::atomic<int> ctas_per_sm[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int per_sm = dev < 64 ? ctas_per_sm[dev].load(std::memory_order_acquire) : 0;
  if (per_sm == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, C::kThreads, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    if (dev < 64) ctas_per_sm[dev].store(per_sm, std::memory_order_release);
  }
  const long long slots = static_cast<long long>(per_sm) * a.num_sms;
  const int grid = static_cast<int>(a.num_items < slots ? a.num_items : slots);
  if (grid < 1) return cudaSuccess;
  kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(kmap, vmap, a);
  return cudaGetLastError();
}

template <int KV, int D, int BS, int NT, bool LP>
static int smem_t() {
  return Cfg<KV, D, BS, NT, LP>::kSmemBytes;
}

int forward_ctas_per_sm(int kv_dtype, int head_size, int block_size, int rows_per_cta) {
  const int smem = forward_smem_bytes(kv_dtype, head_size, block_size, rows_per_cta);
  if (smem <= 0) return 1;
  // 228 KiB of shared memory per SM, 1 KiB reserved per CTA; the launch bounds
  // cap registers at 3 CTAs (one n-tile) or 2 CTAs (two n-tiles) per SM.
  int n = (228 * 1024) / (smem + 1024);
  const int cap = rows_per_cta == 16 ? 2 : 3;
  if (n > cap) n = cap;
  return n < 1 ? 1 : n;
}

template <int KV, int D, int BS>
static int dispatch_rows_smem(int rows) {
  if (rows == 4) return smem_t<KV, D, BS, 1, true>();
  if (rows == 8) return smem_t<KV, D, BS, 1, false>();
  if (rows == 16) return smem_t<KV, D, BS, 2, false>();
  return -1;
}

template <int KV, int D, int BS>
static cudaError_t dispatch_rows(int rows, const CUtensorMap& kmap, const CUtensorMap& vmap,
                                 const FwdArgs& a, cudaStream_t s) {
  if (rows == 4) return launch_t<KV, D, BS, 1, true>(kmap, vmap, a, s);
  if (rows == 8) return launch_t<KV, D, BS, 1, false>(kmap, vmap, a, s);
  if (rows == 16) return launch_t<KV, D, BS, 2, false>(kmap, vmap, a, s);
  return cudaErrorInvalidValue;
}

template <int KV>
static cudaError_t dispatch_shape(int D, int BS, int rows, const CUtensorMap& kmap,
                                  const CUtensorMap& vmap, const FwdArgs& a, cudaStream_t s) {
  if (D == 64 && BS == 16) return dispatch_rows<KV, 64, 16>(rows, kmap, vmap, a, s);
  if (D == 64 && BS == 32) return dispatch_rows<KV, 64, 32>(rows, kmap, vmap, a, s);
  if (D == 128 && BS == 16) return dispatch_rows<KV, 128, 16>(rows, kmap, vmap, a, s);
  if (D == 128 && BS == 32) return dispatch_rows<KV, 128, 32>(rows, kmap, vmap, a, s);
  return cudaErrorInvalidValue;
}

template <int KV>
static int dispatch_shape_smem(int D, int BS, int rows) {
  if (D == 64 && BS == 16) return dispatch_rows_smem<KV, 64, 16>(rows);
  if (D == 64 && BS == 32) return dispatch_rows_smem<KV, 64, 32>(rows);
  if (D == 128 && BS == 16) return dispatch_rows_smem<KV, 128, 16>(rows);
  if (D == 128 && BS == 32) return dispatch_rows_smem<KV, 128, 32>(rows);
  return -1;
}

cudaError_t launch_forward(int kv_dtype, int head_size, int block_size, int rows_per_cta,
                           const CUtensorMap& kmap, const CUtensorMap& vmap, const FwdArgs& a,
                           cudaStream_t stream) {
  switch (kv_dtype) {
    case PA_KV_INT8:
      return dispatch_shape<PA_KV_INT8>(head_size, block_size, rows_per_cta, kmap, vmap, a,
                                        stream);
    case PA_KV_INT4:
      return dispatch_shape<PA_KV_INT4>(head_size, block_size, rows_per_cta, kmap, vmap, a,
                                        stream);
    case PA_KV_FP8_E4M3:
      return dispatch_shape<PA_KV_FP8_E4M3>(head_size, block_size, rows_per_cta, kmap, vmap, a,
                                            stream);
    default:
      return cudaErrorInvalidValue;
  }
}

int forward_smem_bytes(int kv_dtype, int head_size, int block_size, int rows_per_cta) {
  switch (kv_dtype) {
    case PA_KV_INT8:
      return dispatch_shape_smem<PA_KV_INT8>(head_size, block_size, rows_per_cta);
    case PA_KV_INT4:
      return dispatch_shape_smem<PA_KV_INT4>(head_size, block_size, rows_per_cta);
    case PA_KV_FP8_E4M3:
      return dispatch_shape_smem<PA_KV_FP8_E4M3>(head_size, block_size, rows_per_cta);
    default:
      return -1;
  }
}

}  // namespace pa
