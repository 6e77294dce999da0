// pa_attention.cu -- fused paged quantised-KV GQA attention for sm_100a.
//
// Work items.  A unit is one (sequence, KV head, group of query rows); its rows
// are (new token, query head of the group) pairs that read the same keys, so the
// GQA group x new tokens form the N side of a tensor-core tile, keys the M side
// ("swap-AB"), channels the K side.  A unit's key blocks may be split into
// several items (flash decoding).  The kernel is persistent: one CTA per
// resident slot, items handed out by an atomic counter in the workspace.
//
// Per CTA:
//   producer warp : fetches the next item, loads its lengths, bulk-copies its
//                   query rows and both per-channel scale rows into one of two
//                   item slots, then streams its KV blocks (block_table -> two
//                   3-D TMA boxes per block, K rows and V rows of one head) into
//                   a swizzled ring of stages, straight after the previous
//                   item's blocks, so the next item's data lands while the
//                   consumers finish the current one.
//   consumer warps: per item: fold the K scale into the queries, then per 32
//                   keys: ldmatrix (K) -> QK MMA (INT8/INT4 codes straight into
//                   mma.sync m16n8k32 s8/u8 x s8 against four int8 digits of the
//                   folded query, exact int32 accumulation; FP8 codes converted
//                   to fp16 in registers for m16n8k16 against an fp16 high part
//                   plus residual) -> online softmax in the exp2 domain whose
//                   running maximum is only raised (shuffle reduction and
//                   rescale) when a logit exceeds it by more than 2^8 -> P^T to
//                   fp16 with movmatrix -> ldmatrix.trans (V) -> exact
//                   code->fp16 in registers -> mma.sync m16n8k16 into O^T.
// The four consumer warps take alternate 32-key groups and merge (m, l, O)
// through shared memory at the end of an item, where the per-channel V scale is
// applied once.  A split item writes a normalised partial and its log2-sum-exp;
// the last item of a unit to finish (arrival counter in the workspace) merges
// them and resets the counter.
//
// Sources: the per-channel K scale folded into Q with a power-of-two normaliser
// (INT4 paged-KV page, onnxruntime PR 32515, Code analysis 3); INT8 codes kept
// raw and converted to FP16 in registers right before an m16n8k16 MMA with FP32
// accumulation (INT8-KV tensor-core page, onnxruntime PR 33707, Code analysis
// 1); online softmax, masking and the flash-decoding split with a partials
// buffer (GQA GEMV decode page, onnxruntime PR 29216, Code analysis 1-2); the
// grid of units sized by the exact max_query_len (exact max_query_len page,
// onnxruntime PR 28409, Code analysis 2).
#include <math.h>

#include <atomic>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// NT: 8-row n-tiles per CTA (rows = 8 NT).  LOPACK (NT = 1 only): the unit has at
// most 4 rows; B-operand columns 0..3 carry one half of each pair of query parts
// (fp16 high part, or int8 digits 0 and 2) and columns 4..7 the other (residual,
// or digits 1 and 3), halving the QK MMAs.
template <int KV, int D, int BS, int NT, bool LOPACK>
struct Cfg {
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
  // producer group: whole warp iterations, at most kSW blocks per warp, <= 32 lanes
  static constexpr int kItPerGroupRaw = (kSW < 8 ? kSW : 8) / kBPI;
  static constexpr int kGroup = kWarps * kBPI * (kItPerGroupRaw < 1 ? 1 : kItPerGroupRaw);
  static constexpr int kRows = 8 * NT;
  static constexpr bool kImma = (KV != PA_KV_FP8_E4M3);         // QK on int8 tensor cores
  static constexpr int kAcc = LOPACK ? 2 : 4;                   // int32 QK accumulators
  static constexpr int kQRegs = kImma ? (D / 32) * kAcc * 2 : (D / 16) * (LOPACK ? 2 : 4);
  static constexpr int kQElems = D / 4;                         // query channels per thread
  static constexpr int kMaxSplits = 128;
  // shared memory map (all offsets from the 1024-aligned base)
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kQBytes = kRows * D * 2;                 // query rows of one item slot
  static constexpr int kQOff = kRingBytes;                      // 2 slots
  static constexpr int kKsOff = kQOff + 2 * kQBytes;            // k_scale rows, 2 slots
  static constexpr int kVsOff = kKsOff + 2 * D * 4;             // v_scale rows, 2 slots
  static constexpr int kEpiOff = kVsOff + 2 * D * 4;            // per-warp partial outputs,
  static constexpr int kEpiBytes =                              // later the split weights
      (D > kMaxSplits ? D : kMaxSplits) * kRows * 4;
  static constexpr int kBarOff = kEpiOff + kEpiBytes;
  static constexpr int kNumBars = 2 * kStages + 4;              // full, empty, item full/empty
  static constexpr int kDescOff = kBarOff + kNumBars * 8;
  static constexpr int kStatOff = kDescOff + 2 * 64;
  static constexpr int kFlagOff = kStatOff + 2 * kWarps * kRows * 4;
  static constexpr int kSmemBytes = kFlagOff + 16;
  static_assert(kChunks % 2 == 0, "ldmatrix.x4 covers two 16-byte chunks");
  static_assert(kTile % ((kSwzMask + 1) * 128) == 0, "tiles keep the swizzle-atom alignment");
  static_assert(!LOPACK || NT == 1, "residual packing needs a single n-tile");
  static_assert(kTPI == 2, "two 16-key tiles per warp iteration");
  static_assert(kStages <= 64, "stage count");
  static_assert(kGroup <= 32 && kGroup / (kWarps * kBPI) * kBPI <= kSW, "producer group");
  static_assert(kMaxSplits * kRows * 4 <= kEpiBytes, "split weights fit in the epilogue buffer");
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

// Channel of the i-th query value a thread contributes to the QK B operand (the
// thread with index tig in its quad).  It matches the channels ldmatrix hands the
// same thread for the K operand.  Element i = 4 * word + byte (integer caches:
// word = 2 s + r for k32-step s and B register r; FP8: i = 4 s + j for 16-channel
// k-step s and half j).
template <int KV>
__device__ __forceinline__ int q_channel(int i, int tig) {
  const int wd = i >> 2, e = i & 3;
  if constexpr (KV == PA_KV_INT8) {
    return 32 * (wd >> 1) + 16 * (wd & 1) + 4 * tig + e;
  } else if constexpr (KV == PA_KV_INT4) {
    return 32 * (wd >> 1) + 8 * tig + 2 * e + (wd & 1);
  } else {
    return 16 * wd + 4 * tig + e;
  }
}

// First of the two adjacent output dims held by M rows g / g+8 of PV m-tile mt.
template <int KV>
__device__ __forceinline__ int out_dim(int mt, int g) {
  if constexpr (KV == PA_KV_INT4) return 32 * (mt >> 1) + 4 * g + 2 * (mt & 1);
  return 16 * mt + 2 * g;
}

// One bulk copy (global -> shared) completing on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Rows, keys and block range of work item w, from the device lengths of its
// sequence.  Returns false (and leaves d.valid = 0) when the item has no work:
// no new tokens, fewer rows than its row group, or a split past the last block.
template <int BS>
__device__ __forceinline__ bool decode_item(const FwdArgs& a, int rows_cta, int w, int q0,
                                            int q1, int Lb, ItemDesc& d) {
  const int u = w / a.num_splits;
  d.valid = 0;
  d.split = w % a.num_splits;
  d.rg = u % a.num_row_groups;
  d.kv = (u / a.num_row_groups) % a.Hk;
  d.b = u / (a.num_row_groups * a.Hk);
  const int qb = q1 - q0;
  if (q0 < 0 || qb < 0 || qb > Lb || q0 + qb > a.total_q ||
      static_cast<long long>(Lb) > static_cast<long long>(a.maxb) * BS) {
    record_error(a.err, PA_DEVERR_BAD_LENGTH);
    return false;
  }
  const int R = qb * a.G;  // rows of (b, kv): row r = token (r / G), head kv*G + r % G
  d.row0 = d.rg * rows_cta;
  if (d.row0 >= R) return false;
  d.row_end = min(R, d.row0 + rows_cta);
  d.q0 = q0;
  d.Lb = Lb;
  d.past = Lb - qb;
  const int i_first = d.row0 / a.G, i_last = (d.row_end - 1) / a.G;
  d.kmax = a.causal ? d.past + i_last + 1 : Lb;    // keys seen by some row
  d.kfull = a.causal ? d.past + i_first + 1 : Lb;  // keys seen by every row
  const int nblk = (d.kmax + BS - 1) / BS;
  d.nsplit = (nblk + a.blocks_per_split - 1) / a.blocks_per_split;
  if (d.split >= d.nsplit) return false;
  d.blk_begin = d.split * a.blocks_per_split;
  d.nloc = min(nblk, d.blk_begin + a.blocks_per_split) - d.blk_begin;
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

template <int KV, int D, int BS, int NT, bool LOPACK>
__global__ void __launch_bounds__(Cfg<KV, D, BS, NT, LOPACK>::kThreads)
    pa_fwd_kernel(const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap, const FwdArgs a) {
  using C = Cfg<KV, D, BS, NT, LOPACK>;
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
  float* sm_m = reinterpret_cast<float*>(smem + C::kStatOff);
  float* sm_l = sm_m + C::kWarps * C::kRows;
  int* sm_flag = reinterpret_cast<int*>(smem + C::kFlagOff);
  float* epi = reinterpret_cast<float*>(smem + C::kEpiOff);
  float* wts = epi;  // split merge weights, once the per-warp outputs are consumed

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int rows_cta = LOPACK ? 4 : C::kRows;

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
    auto fetch = [&]() {
      int w = 0;
      if (lane == 0) w = static_cast<int>(atomicAdd(a.work, 1u));
      return __shfl_sync(0xffffffffu, w, 0);
    };
    int uses[2] = {0, 0};
    int slot = 0;
    // Blocks handed to each consumer warp so far: warp w's k-th block lives in
    // stage w * kSW + k % kSW of its own sub-ring, round k / kSW.
    int cnt[C::kWarps] = {0, 0, 0, 0};
    bool ok = true;
    int w = fetch();
    while (ok) {
      ItemDesc d;
      d.valid = 0;
      while (w < a.num_items) {
        const int b = (w / a.num_splits) / (a.num_row_groups * a.Hk);
        int v = 0;
        if (lane == 0) v = a.cu_seqlens_q[b];
        else if (lane == 1) v = a.cu_seqlens_q[b + 1];
        else if (lane == 2) v = a.seqlens_k[b];
        const int q0 = __shfl_sync(0xffffffffu, v, 0);
        const int q1 = __shfl_sync(0xffffffffu, v, 1);
        const int Lb = __shfl_sync(0xffffffffu, v, 2);
        if (decode_item<BS>(a, rows_cta, w, q0, q1, Lb, d)) break;
        w = fetch();
      }
      // publish the item (or the end marker) in the next slot
      if (lane == 0) {
        if (uses[slot] > 0 && !mbar_wait(item_empty(slot), (uses[slot] - 1) & 1)) {
          record_error(a.err, PA_DEVERR_TIMEOUT);
          ok = false;
        } else {
          descs[slot] = d;
          if (d.valid) {
            const uint32_t row_bytes = D * 2;
            const uint32_t total =
                static_cast<uint32_t>(d.row_end - d.row0) * row_bytes + 2 * D * 4;
            mbar_arrive_expect_tx(item_full(slot), total);
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
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ++uses[slot];
      if (!ok || !d.valid) break;
      const int w_next = fetch();  // overlaps with streaming this item

      // Blocks go out in groups of kGroup (whole warp iterations, at most kSW
      // blocks of any warp, so every block of a group has its own stage): lane j
      // waits for its stage to be released, arms it and issues the two boxes,
      // all lanes in parallel.  Item block lb belongs to warp (lb / kBPI) % 4,
      // the same split the consumers use.
      constexpr int kGroup = C::kGroup;
      const int32_t* bt = a.block_table + static_cast<size_t>(d.b) * a.maxb + d.blk_begin;
      for (int base = 0; base < d.nloc && ok; base += kGroup) {
        const int lb = base + lane;
        bool mine_ok = true;
        if (lane < kGroup && lb < d.nloc) {
          int phys = __ldg(bt + lb);
          if (phys < 0 || phys >= a.num_blocks) {
            record_error(a.err, PA_DEVERR_BAD_BLOCK);
            phys = a.num_blocks;  // out-of-range box: TMA fills zeros, nothing faults
          }
          const int wq = (lb / C::kBPI) % C::kWarps;
          const int k = cnt[wq] + (lb / (C::kWarps * C::kBPI)) * C::kBPI + lb % C::kBPI;
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
        ok = __all_sync(0xffffffffu, mine_ok);
        if (!ok && lane == 0) record_error(a.err, PA_DEVERR_TIMEOUT);
      }
#pragma unroll
      for (int wq = 0; wq < C::kWarps; ++wq) cnt[wq] += warp_blocks<C::kBPI>(d.nloc, wq);
      slot ^= 1;
      w = w_next;
    }
    // Leave no copy in flight: wait for the last box of every stage, all within
    // one bounded window (the consumers normally consumed them already).
    if (lane == 0) {
      const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
      bool fine = true;
      for (int wq = 0; wq < C::kWarps; ++wq)
        for (int j = 0; fine && j < C::kSW && j < cnt[wq]; ++j) {
          const int last_round = (cnt[wq] - 1 - j) / C::kSW;
          fine = mbar_wait_until(full_bar(wq * C::kSW + j), last_round & 1, deadline);
        }
      if (!fine) record_error(a.err, PA_DEVERR_TIMEOUT);
      // The last CTA to finish rewinds the work counter for the next call.
      if (atomicAdd(a.work + 1, 1u) == gridDim.x - 1) {
        a.work[0] = 0u;
        a.work[1] = 0u;
      }
    }
    return;
  }

  // ======================================================== consumer warps
  int uses[2] = {0, 0};
  int slot = 0;
  int kc = 0;  // blocks this warp consumed so far: its k-th block is in stage
               // warp * kSW + k % kSW of its own sub-ring, round k / kSW
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
    const int blk_begin = d.blk_begin, nloc = d.nloc, Lb = d.Lb, nsplit = d.nsplit;
    const float* sks = reinterpret_cast<const float*>(smem + C::kKsOff) + slot * D;
    const float* svs = reinterpret_cast<const float*>(smem + C::kVsOff) + slot * D;
    bool alive = true;

    // ---- prologue: fold the K scale into the queries.  q'[d] = q[d] k_scale[d] /
    // 2^e_kv (2^e_kv: power of two of max |k_scale| of this head), then a second
    // power of two per row keeps |q'| < 1 for any finite input; both powers move
    // into the per-row logit multiplier c (exp2 domain).
    float ksmax = 0.f;
  #pragma unroll
    for (int d = lane; d < D; d += 32) ksmax = fmaxf(ksmax, fabsf(sks[d]));
  #pragma unroll
    for (int o = 16; o > 0; o >>= 1) ksmax = fmaxf(ksmax, __shfl_xor_sync(0xffffffffu, ksmax, o));
    if (!isfinite(ksmax) && warp == 0 && lane == 0) record_error(a.err, PA_DEVERR_BAD_SCALE);
    int e_kv = 0;
    (void)frexpf(ksmax, &e_kv);
    const float f_kv = ldexpf(1.f, -e_kv);

    // Query operand.  Integer caches (INT8/INT4): q'' = 64 q' is split into four
    // signed int8 digits, q'' = d0 + d1 2^-7 + d2 2^-14 + d3 2^-21 (residual below
    // 2^-22), each digit a B operand of an exact int8 x int8 -> int32 MMA whose A
    // operand is the raw cache code (INT4 as code + 8, corrected exactly with the
    // digit sums).  FP8 caches: q' as an fp16 high part plus its fp16 residual.
    // With LOPACK the second half of each pair rides in MMA columns 4..7.
    uint32_t qf[NT][C::kQRegs];
    float cw[NT][2][2];  // per accumulator column j: combine weights
    int qoff[NT][2][2];  // per accumulator column j: integer offsets (magic - bias)
    int lim[NT][2];
    const __half* sq16 = reinterpret_cast<const __half*>(smem + C::kQOff + slot * C::kQBytes);
    const __nv_bfloat16* sqbf = reinterpret_cast<const __nv_bfloat16*>(sq16);
  #pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int rl = LOPACK ? (g & 3) : nt * 8 + g;  // local row of B-operand column g
      const bool valid = row0 + rl < row_end;
      float w[C::kQElems];
      float rmax = 0.f;
  #pragma unroll
      for (int i = 0; i < C::kQElems; ++i) {
        const int ch = q_channel<KV>(i, tig);
        float x = 0.f;
        if (valid)
          x = a.q_bf16 ? __bfloat162float(sqbf[rl * D + ch]) : __half2float(sq16[rl * D + ch]);
        w[i] = x * (sks[ch] * f_kv);
        rmax = fmaxf(rmax, fabsf(w[i]));
      }
      rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 1));
      rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 2));
      int e_q = 0;
      (void)frexpf(rmax, &e_q);
      const float c_mine = ldexpf(a.sm_scale_log2, e_kv + e_q);
      if constexpr (C::kImma) {
        const float f64 = ldexpf(1.f, 6 - e_q);
        int dsum[4] = {0, 0, 0, 0};
        uint32_t words[4][C::kQElems / 4];
  #pragma unroll
        for (int wd = 0; wd < C::kQElems / 4; ++wd)
  #pragma unroll
          for (int dg = 0; dg < 4; ++dg) words[dg][wd] = 0u;
  #pragma unroll
        for (int i = 0; i < C::kQElems; ++i) {
          float r = w[i] * f64;  // |r| < 64
          int dg_val[4];
  #pragma unroll
          for (int dg = 0; dg < 4; ++dg) {
            const float dgt = rintf(r);
            dg_val[dg] = static_cast<int>(dgt);
            r = (r - dgt) * 128.f;
          }
  #pragma unroll
          for (int dg = 0; dg < 4; ++dg) {
            dsum[dg] += dg_val[dg];
            words[dg][i / 4] |= (static_cast<uint32_t>(dg_val[dg]) & 0xFFu) << (8 * (i % 4));
          }
        }
  #pragma unroll
        for (int dg = 0; dg < 4; ++dg) {
          dsum[dg] += __shfl_xor_sync(0xffffffffu, dsum[dg], 1);
          dsum[dg] += __shfl_xor_sync(0xffffffffu, dsum[dg], 2);
        }
        // qf layout: [k32 step s][accumulator i][b register r]
  #pragma unroll
        for (int s = 0; s < D / 32; ++s)
  #pragma unroll
          for (int i = 0; i < C::kAcc; ++i)
  #pragma unroll
            for (int r = 0; r < 2; ++r) {
              // LOPACK: accumulator i carries digits (i=0: 0|1, i=1: 2|3), the odd
              // digit in columns 4..7 (lanes with g >= 4)
              const int dg = LOPACK ? (2 * i + (g >= 4 ? 1 : 0)) : i;
              qf[nt][(s * C::kAcc + i) * 2 + r] = words[dg][s * 2 + r];
            }
        constexpr int kMagic = 0x4B400000;
        const int kbias = (KV == PA_KV_INT4) ? 8 : 0;  // A operand holds code + 8
  #pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int col = 2 * tig + j;  // accumulator column held by this thread
          const int src = col * 4;  // lanes with g = col supplied this column
          if constexpr (LOPACK) {
            // lane g = col supplied this column: digits 0|2 of row col (col < 4) or
            // 1|3 of row col - 4; every lane holds all four digit sums of its row
            const int sA = __shfl_sync(0xffffffffu, dsum[0], src);
            const int sA1 = __shfl_sync(0xffffffffu, dsum[1], src);
            const int sB = __shfl_sync(0xffffffffu, dsum[2], src);
            const int sB1 = __shfl_sync(0xffffffffu, dsum[3], src);
            const bool odd = col >= 4;
            qoff[nt][j][0] = kMagic - kbias * (odd ? sA1 : sA);
            qoff[nt][j][1] = kMagic - kbias * (odd ? sB1 : sB);
            const int rr = col & 3;
            const float cr = __shfl_sync(0xffffffffu, c_mine, rr * 4) * (1.f / 64.f);
            // own value v = digit_even_or_odd + 2^-14 * next; S = v_even + 2^-7 v_odd
            cw[nt][j][0] = odd ? cr * (1.f / 128.f) : cr;  // weight of own v
            cw[nt][j][1] = odd ? cr : cr * (1.f / 128.f);  // weight of partner v
          } else {
            const int s0 = __shfl_sync(0xffffffffu, dsum[0], src);
            const int s1 = __shfl_sync(0xffffffffu, dsum[1], src);
            const int s2 = __shfl_sync(0xffffffffu, dsum[2], src);
            const int s3 = __shfl_sync(0xffffffffu, dsum[3], src);
            qoff[nt][j][0] = kbias * (s0 * 128 + s1);
            qoff[nt][j][1] = kbias * (s2 * 128 + s3);
            const float cr = __shfl_sync(0xffffffffu, c_mine, src) * (1.f / 64.f);
            cw[nt][j][0] = cr * (1.f / 128.f);
            cw[nt][j][1] = cr * (1.f / 2097152.f);  // 2^-21
          }
        }
      } else {
        const float f_q = ldexpf(1.f, -e_q);
  #pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          float hi[4], lo[4];
  #pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float xn = w[s * 4 + j] * f_q;
            hi[j] = __half2float(__float2half_rn(xn));
            lo[j] = xn - hi[j];
          }
          if constexpr (LOPACK) {
            const bool use_lo = g >= 4;
            qf[nt][s * 2 + 0] = pack_f32x2_to_h2(use_lo ? lo[0] : hi[0], use_lo ? lo[1] : hi[1]);
            qf[nt][s * 2 + 1] = pack_f32x2_to_h2(use_lo ? lo[2] : hi[2], use_lo ? lo[3] : hi[3]);
          } else {
            qf[nt][s * 4 + 0] = pack_f32x2_to_h2(hi[0], hi[1]);
            qf[nt][s * 4 + 1] = pack_f32x2_to_h2(hi[2], hi[3]);
            qf[nt][s * 4 + 2] = pack_f32x2_to_h2(lo[0], lo[1]);
            qf[nt][s * 4 + 3] = pack_f32x2_to_h2(lo[2], lo[3]);
          }
        }
  #pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int rr = LOPACK ? ((2 * tig + j) & 3) : 2 * tig + j;
          cw[nt][j][0] = __shfl_sync(0xffffffffu, c_mine, rr * 4);
          cw[nt][j][1] = 0.f;
          qoff[nt][j][0] = qoff[nt][j][1] = 0;
        }
      }
  #pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int rr = LOPACK ? ((2 * tig + j) & 3) : nt * 8 + 2 * tig + j;
        lim[nt][j] = (row0 + rr < row_end && a.causal) ? past + (row0 + rr) / a.G : kmax - 1;
      }
    }

    float o[NT][C::kMTiles][4];
    float m_run[NT][2], l_run[NT][2];  // l_run: sum of the fp16-rounded P the MMA used
  #pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
  #pragma unroll
      for (int mt = 0; mt < C::kMTiles; ++mt)
  #pragma unroll
        for (int e = 0; e < 4; ++e) o[nt][mt][e] = 0.f;
      m_run[nt][0] = m_run[nt][1] = -INFINITY;
      l_run[nt][0] = l_run[nt][1] = 0.f;
    }

    // ldmatrix lane addressing: matrix (lane >> 3) covers rows (lane & 7) + 8 * (m & 1)
    // of a 16-row key tile and chunk (2 cp + (m >> 1)).
    const int lm = lane >> 3;
    const int ld_row = (lane & 7) + 8 * (lm & 1);
    const int ld_chunk = lm >> 1;

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

      float x[C::kTPI][NT][4];  // logits (log2 units), then probabilities
  #pragma unroll
      for (int t = 0; t < C::kTPI; ++t) {
        if (t >= ntiles) {
  #pragma unroll
          for (int nt = 0; nt < NT; ++nt)
  #pragma unroll
            for (int e = 0; e < 4; ++e) x[t][nt][e] = -INFINITY;
          continue;
        }
        const int bi = t / C::kKeyTiles, kt = t % C::kKeyTiles;
        const uint32_t kbase = smem_u32(k_tile(warp * C::kSW + (kc + bi) % C::kSW));
        const int key0 = (blk_begin + lb0 + bi) * BS + kt * 16;
        const bool need_mask = key0 + 16 > kfull;
        if constexpr (C::kImma) {
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
                a0 = r[0]; a1 = r[1]; a2 = r[2]; a3 = r[3];  // 32 channels, no conversion
                s = cp;
              } else {
                const uint32_t x0 = r[2 * h], x1 = r[2 * h + 1];  // rows g, g+8 of chunk 2cp+h
                a0 = i4lo_to_u8x4(x0);
                a1 = i4lo_to_u8x4(x1);
                a2 = i4hi_to_u8x4(x0);
                a3 = i4hi_to_u8x4(x1);
                s = 2 * cp + h;
              }
  #pragma unroll
              for (int nt = 0; nt < NT; ++nt)
  #pragma unroll
                for (int i = 0; i < C::kAcc; ++i)
                  imma_16832<KV == PA_KV_INT4>(acc[i][nt], a0, a1, a2, a3,
                                               qf[nt][(s * C::kAcc + i) * 2],
                                               qf[nt][(s * C::kAcc + i) * 2 + 1]);
            }
          }
  #pragma unroll
          for (int nt = 0; nt < NT; ++nt)
  #pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = e & 1;
              float xv;
              if constexpr (LOPACK) {
                const float f1 = int_to_float_exact(acc[0][nt][e], qoff[nt][j][0]);
                const float f2 = int_to_float_exact(acc[1][nt][e], qoff[nt][j][1]);
                const float v = fmaf(f2, 1.f / 16384.f, f1);
                const float pv = __shfl_xor_sync(0xffffffffu, v, 2);
                xv = fmaf(pv, cw[nt][j][1], v * cw[nt][j][0]);
              } else {
                const int A = acc[0][nt][e] * 128 + acc[1][nt][e] - qoff[nt][j][0];
                const int B = acc[2][nt][e] * 128 + acc[3][nt][e] - qoff[nt][j][1];
                xv = fmaf(__int2float_rn(B), cw[nt][j][1], __int2float_rn(A) * cw[nt][j][0]);
              }
              if (need_mask && key0 + g + (e >> 1) * 8 > lim[nt][j]) xv = -INFINITY;
              x[t][nt][e] = xv;
            }
        } else {
          float sacc[NT][4], sres[NT][4];
  #pragma unroll
          for (int nt = 0; nt < NT; ++nt)
  #pragma unroll
            for (int e = 0; e < 4; ++e) sacc[nt][e] = sres[nt][e] = 0.f;
  #pragma unroll
          for (int cp = 0; cp < C::kChunks / 2; ++cp) {
            uint32_t r[4];
            const uint32_t off = (kt * 16 + ld_row) * C::kCHS + (2 * cp + ld_chunk) * 16;
            ldsm_x4(kbase + swz<C::kSwzMask>(off), r);
  #pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int s = 2 * cp + h;  // 16-channel k-step
              uint32_t a0, a1, a2, a3;
              e4m3x4_to_h2x2(r[2 * h], a0, a2);      // row g: channels +0,1 | +2,3
              e4m3x4_to_h2x2(r[2 * h + 1], a1, a3);  // row g+8
  #pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                if constexpr (LOPACK) {
                  mma_16816(sacc[nt], a0, a1, a2, a3, qf[nt][s * 2], qf[nt][s * 2 + 1]);
                } else {
                  mma_16816(sacc[nt], a0, a1, a2, a3, qf[nt][s * 4], qf[nt][s * 4 + 1]);
                  mma_16816(sres[nt], a0, a1, a2, a3, qf[nt][s * 4 + 2], qf[nt][s * 4 + 3]);
                }
              }
            }
          }
  #pragma unroll
          for (int nt = 0; nt < NT; ++nt)
  #pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = e & 1;
              float sv = sacc[nt][e];
              if constexpr (LOPACK)
                sv += __shfl_xor_sync(0xffffffffu, sv, 2);  // high part + residual part
              else
                sv += sres[nt][e];
              float xv = sv * cw[nt][j][0];
              if (need_mask && key0 + g + (e >> 1) * 8 > lim[nt][j]) xv = -INFINITY;
              x[t][nt][e] = xv;
            }
        }
      }

      // ---------------- online softmax with a lazily raised running max
  #pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
  #pragma unroll
        for (int j = 0; j < 2; ++j) {
          float lmx = -INFINITY;
  #pragma unroll
          for (int t = 0; t < C::kTPI; ++t) lmx = fmaxf(lmx, fmaxf(x[t][nt][j], x[t][nt][j + 2]));
          const bool raise = lmx > m_run[nt][j] + 8.f;
          if (__any_sync(0xffffffffu, raise)) {
            lmx = fmaxf(lmx, __shfl_xor_sync(0xffffffffu, lmx, 4));
            lmx = fmaxf(lmx, __shfl_xor_sync(0xffffffffu, lmx, 8));
            lmx = fmaxf(lmx, __shfl_xor_sync(0xffffffffu, lmx, 16));
            if (lmx > m_run[nt][j]) {
              const float alpha = fast_exp2(m_run[nt][j] - lmx);  // 0 when m_run = -inf
              m_run[nt][j] = lmx;
              l_run[nt][j] *= alpha;
  #pragma unroll
              for (int mt = 0; mt < C::kMTiles; ++mt) {
                o[nt][mt][j] *= alpha;
                o[nt][mt][j + 2] *= alpha;
              }
            }
          }
          const float m_ref = (m_run[nt][j] == -INFINITY) ? 0.f : m_run[nt][j];
  #pragma unroll
          for (int t = 0; t < C::kTPI; ++t) {
            x[t][nt][j] = fast_exp2(x[t][nt][j] - m_ref);  // <= 2^8: safe range for fp16
            x[t][nt][j + 2] = fast_exp2(x[t][nt][j + 2] - m_ref);
          }
        }
      }

      // ---------------- O^T[dim, row] += V^T P^T, per key tile
  #pragma unroll
      for (int t = 0; t < C::kTPI; ++t) {
        if (t >= ntiles) continue;
        const int bi = t / C::kKeyTiles, kt = t % C::kKeyTiles;
        const uint32_t vbase = smem_u32(v_tile(warp * C::kSW + (kc + bi) % C::kSW));
        // P^T as the B operand: (key g; rows 2tig, 2tig+1) -> (keys 2tig, 2tig+1; row g);
        // l_run accumulates exactly the fp16 values the MMA consumes.
        uint32_t pb[NT][2];
  #pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint32_t p01 = pack_f32x2_to_h2(x[t][nt][0], x[t][nt][1]);
          const uint32_t p23 = pack_f32x2_to_h2(x[t][nt][2], x[t][nt][3]);
          const __half2 h01 = u2h2(p01), h23 = u2h2(p23);
          l_run[nt][0] += __low2float(h01) + __low2float(h23);
          l_run[nt][1] += __high2float(h01) + __high2float(h23);
          pb[nt][0] = movmatrix_trans(p01);
          pb[nt][1] = movmatrix_trans(p23);
        }
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
                // fp16 1024 + (code + 128): the constant 1152 per key is removed once
                // at the end as 1152 * sum(P)
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
                const uint32_t zl = lo >> (8 * hh), zh = hi >> (8 * hh);
                a0 = i4lo_to_h2(zl);
                a1 = i4hi_to_h2(zl);
                a2 = i4lo_to_h2(zh);
                a3 = i4hi_to_h2(zh);
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

    // ======================================================== merge the warps
    // Accumulator column 2 tig + j holds local row nt*8 + 2 tig + j (with LOPACK:
    // row (2 tig + j) & 3, columns 4..7 duplicating rows 0..3, so only tig < 2
    // writes).
    const bool writer = !LOPACK || tig < 2;
  #pragma unroll
    for (int nt = 0; nt < NT; ++nt)
  #pragma unroll
      for (int j = 0; j < 2; ++j) {
        float l = l_run[nt][j];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        l_run[nt][j] = l;
        if (g == 0 && writer) {
          sm_m[warp * C::kRows + nt * 8 + 2 * tig + j] = m_run[nt][j];
          sm_l[warp * C::kRows + nt * 8 + 2 * tig + j] = l;
        }
      }
    consumer_sync();
    // The warps' rescaled outputs are summed into one [rows, D] buffer, warp 3
    // first, then 2, 1, 0 (a fixed order: results are bitwise reproducible).
    for (int wsum = C::kWarps - 1; wsum >= 0; --wsum) {
      if (warp == wsum && writer) {
  #pragma unroll
        for (int nt = 0; nt < NT; ++nt)
  #pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int row = nt * 8 + 2 * tig + j;
            float M = -INFINITY;
  #pragma unroll
            for (int w = 0; w < C::kWarps; ++w) M = fmaxf(M, sm_m[w * C::kRows + row]);
            const float f = (m_run[nt][j] == -INFINITY) ? 0.f : fast_exp2(m_run[nt][j] - M);
            // INT8 V entered the MMA as fp16 (1152 + code): remove 1152 * sum(P)
            const float vbias = (KV == PA_KV_INT8) ? 1152.f * l_run[nt][j] : 0.f;
  #pragma unroll
            for (int mt = 0; mt < C::kMTiles; ++mt) {
              const int d = out_dim<KV>(mt, g);
              float2* dst = reinterpret_cast<float2*>(epi + row * D + d);
              float2 v = make_float2((o[nt][mt][j] - vbias) * f, (o[nt][mt][j + 2] - vbias) * f);
              if (wsum != C::kWarps - 1) {
                const float2 prev = *dst;
                v.x += prev.x;
                v.y += prev.y;
              }
              *dst = v;
            }
          }
      }
      consumer_sync();
    }

    const int nthr = C::kWarps * 32;
    const int nrows = row_end - row0;
    for (int idx = threadIdx.x; idx < nrows * (D / 2); idx += nthr) {
      const int row = idx / (D / 2);
      const int d = (idx % (D / 2)) * 2;
      float M = -INFINITY;
  #pragma unroll
      for (int w = 0; w < C::kWarps; ++w) M = fmaxf(M, sm_m[w * C::kRows + row]);
      float L = 0.f;
  #pragma unroll
      for (int w = 0; w < C::kWarps; ++w) {
        const float mw = sm_m[w * C::kRows + row];
        if (mw != -INFINITY) L += sm_l[w * C::kRows + row] * fast_exp2(mw - M);
      }
      const float2 sv = *reinterpret_cast<const float2*>(epi + row * D + d);
      const float s0 = sv.x, s1 = sv.y;
      const float inv = (L > 0.f) ? 1.f / L : 0.f;
      const float o0 = s0 * inv * svs[d];
      const float o1 = s1 * inv * svs[d + 1];
      const int r = row0 + row;
      const size_t orow = static_cast<size_t>(q0 + r / a.G) * a.H + kv * a.G + r % a.G;
      if (nsplit == 1) {
        if (a.out_bf16)
          *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(a.out) + orow * D +
                                             d) = __floats2bfloat162_rn(o0, o1);
        else
          *reinterpret_cast<__half2*>(reinterpret_cast<__half*>(a.out) + orow * D + d) =
              __floats2half2_rn(o0, o1);
      } else {
        const size_t prow = static_cast<size_t>(split) * a.total_q * a.H + orow;
        *reinterpret_cast<float2*>(a.o_part + prow * D + d) = make_float2(o0, o1);
        if (d == 0) a.lse_part[prow] = (L > 0.f) ? M + __log2f(L) : -INFINITY;
      }
    }
    if (nsplit > 1) {
      // ---- split merge: publish this split and count arrivals; the last item
      // of the unit merges all splits (log2-sum-exp weights) and rewinds the
      // counter for the next call.
      __threadfence();
      consumer_sync();
      uint32_t* counter =
          a.counters + (static_cast<size_t>(b) * a.Hk + kv) * a.num_row_groups + rg;
      if (threadIdx.x == 0) {
        const uint32_t prev = atomicAdd(counter, 1u);
        *sm_flag = (prev == static_cast<uint32_t>(nsplit - 1)) ? 1 : 0;
      }
      consumer_sync();
      if (*sm_flag) {
        __threadfence();
        const size_t stride = static_cast<size_t>(a.total_q) * a.H;
        const int S = nsplit;
        // 1) every (split, row) log2-sum-exp, loaded in parallel
        for (int idx = threadIdx.x; idx < S * nrows; idx += nthr) {
          const int s = idx / nrows, row = idx % nrows;
          const int r = row0 + row;
          const size_t orow = static_cast<size_t>(q0 + r / a.G) * a.H + kv * a.G + r % a.G;
          wts[s * C::kRows + row] = __ldcg(a.lse_part + s * stride + orow);
        }
        consumer_sync();
        // 2) per row: weights 2^(lse_s - max) / sum
        for (int row = threadIdx.x; row < nrows; row += nthr) {
          float M = -INFINITY;
          for (int s = 0; s < S; ++s) M = fmaxf(M, wts[s * C::kRows + row]);
          float sum = 0.f;
          for (int s = 0; s < S; ++s) {
            const float ls = wts[s * C::kRows + row];
            const float wgt = (ls == -INFINITY) ? 0.f : fast_exp2(ls - M);
            wts[s * C::kRows + row] = wgt;
            sum += wgt;
          }
          const float inv = sum > 0.f ? 1.f / sum : 0.f;
          for (int s = 0; s < S; ++s) wts[s * C::kRows + row] *= inv;
        }
        consumer_sync();
        // 3) weighted sum of the partials, eight splits in flight per thread
        for (int idx = threadIdx.x; idx < nrows * (D / 2); idx += nthr) {
          const int row = idx / (D / 2);
          const int dd = (idx % (D / 2)) * 2;
          const int r = row0 + row;
          const size_t orow = static_cast<size_t>(q0 + r / a.G) * a.H + kv * a.G + r % a.G;
          const float* base = a.o_part + orow * D + dd;
          float s0 = 0.f, s1 = 0.f;
          for (int s8 = 0; s8 < S; s8 += 8) {
            float2 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
              v[u] = (s8 + u < S)
                         ? __ldcg(reinterpret_cast<const float2*>(base + (s8 + u) * stride * D))
                         : make_float2(0.f, 0.f);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              if (s8 + u < S) {
                const float wgt = wts[(s8 + u) * C::kRows + row];
                s0 += wgt * v[u].x;
                s1 += wgt * v[u].y;
              }
            }
          }
          if (a.out_bf16)
            *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(a.out) +
                                               orow * D + dd) = __floats2bfloat162_rn(s0, s1);
          else
            *reinterpret_cast<__half2*>(reinterpret_cast<__half*>(a.out) + orow * D + dd) =
                __floats2half2_rn(s0, s1);
        }
        if (threadIdx.x == 0) *counter = 0u;  // ready for the next call
      }
    }
    // the item slot (query rows, scales, descriptor) may be refilled
    consumer_sync();
    if (threadIdx.x == 0) mbar_arrive(item_empty(slot));
    slot ^= 1;
  }
}

template <int KV, int D, int BS, int NT, bool LOPACK>
static cudaError_t launch_t(const CUtensorMap& kmap, const CUtensorMap& vmap, FwdArgs a,
                            cudaStream_t stream) {
  using C = Cfg<KV, D, BS, NT, LOPACK>;
  auto kern = pa_fwd_kernel<KV, D, BS, NT, LOPACK>;
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

template <int KV, int D, int BS, int NT, bool LOPACK>
static int smem_t() {
  return Cfg<KV, D, BS, NT, LOPACK>::kSmemBytes;
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
