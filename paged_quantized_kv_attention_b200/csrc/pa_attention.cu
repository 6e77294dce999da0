// pa_attention.cu -- fused paged quantised-KV GQA attention for sm_100a.
//
// A call is three kernels chained by programmatic dependent launch:
//   pa_prep_kernel    folds each KV head's k_scale into its query rows and stores
//                     every consumer lane's B-operand words (query digits or fp16
//                     parts) and the rows' logit multipliers in the workspace,
//                     once per (sequence, KV head, row group) unit;
//   pa_fwd_kernel     the fused, persistent attention kernel (below);
//   pa_combine_kernel the log-sum-exp merge of split partials (only when the
//                     plan splits the KV).
//
// Work items.  An item is (sequence, group of 4 KV heads, group of query rows,
// KV split).  The rows of one head are the (new token, query head of the GQA
// group) pairs that read that head's keys; they form the N side of the
// tensor-core tiles, keys the M side ("swap-AB"), channels the K side.  A
// sequence with n KV blocks is cut into ceil(n / T) equal splits (flash
// decoding), T chosen by the planner so that the items fill the resident CTAs.
// Items are numbered densely over the sequences with new tokens: the producer
// warp of every CTA computes the per-sequence item counts and their prefix sums
// once, from the device lengths, into a shared-memory table.  The kernel is
// persistent: CTA i starts with item i and then pulls items from an atomic
// counter in the workspace.
//
// Per CTA, one producer warp and four consumer warps, consumer warp w owning KV
// head 4 hg + w of the item:
//   producer : per item, streams the KV in stages of 16 tokens: one 3-D TMA box
//              (channels x 16 tokens x 4 heads, heads outermost in shared
//              memory) for K and one for V into an mbarrier ring.  Producer lane
//              l owns ring stage l and refills it as soon as all four consumer
//              warps have released it; when no lane can issue, the warp sleeps
//              on its oldest pending stage.
//   consumers: per item, each warp loads its head's fragments (after the
//              pre-pass grid completes, for the first item), then for every
//              stage: ldmatrix (its head's K rows) -> QK on the tensor cores ->
//              online softmax (exp2 domain; the running maximum is raised only
//              when a logit exceeds it by more than 2^8) -> P^T in fp16 ->
//              ldmatrix.trans (V) -> code -> fp16 -> PV MMA.  With one n-tile the
//              next stage's QK MMAs are issued before this stage's softmax and
//              PV.  At the end the warp applies the V scale and stores its head's
//              rows (and, on request, their log-sum-exps), or writes an fp16
//              split partial in code units, its log2-sum-exp and the row's split
//              count for the combine.  No consumer barrier: the warps never wait
//              on each other.
//
// QK arithmetic.  INT8 and INT4 caches: the folded query q'' = q' 2^(6 - e_q)
// (|q''| < 64) is split into signed int8 digits q'' = d0 + d1 2^-7 + d2 2^-14
// (+ d3 2^-21), each the B operand of an exact mma.sync m16n8k32 s8 x s8 -> s32
// whose A operand is the raw cache byte (INT4: the nibble shifted into the high
// half of a byte, 16 x code).  FP8 caches: codes -> fp16 in registers, q' as an
// fp16 high part plus an fp16 residual.  With at most 4 rows per head, MMA column
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
#include <type_traits>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

constexpr uint32_t kFull = 0xffffffffu;
constexpr uint32_t kOnesH2 = 0x3C003C00u;  // fp16x2 (1, 1)

// NT: 8-column n-tiles per head (rows = 8 NT).  LP: at most 4 rows per head; MMA
// column n carries row n / 2 (QK: the two halves of a digit/part pair; PV: the
// row twice).
template <int KV, int D, int BS, int NT, bool LP>
struct Cfg {
  static_assert(!LP || NT == 1, "row-pair packing uses one n-tile");
  static constexpr bool kInt = (KV != PA_KV_FP8_E4M3);
  static constexpr int kCHS = (KV == PA_KV_INT4) ? D / 2 : D;  // cache bytes per row
  static constexpr int kHP = kHeadsPerItem;                     // KV heads per item
  static constexpr int kTok = 16;                               // tokens per stage
  static constexpr int kSPB = BS / kTok;                        // stages per cache block
  static constexpr int kHeadTile = kTok * kCHS;                 // one head's rows of a stage
  static constexpr int kKTile = kHP * kHeadTile;                // K (or V) part of a stage
  static constexpr int kStageBytes = 2 * kKTile;
  static constexpr int kChunks = kCHS / 16;                     // 16-byte chunks per row
  static constexpr int kSwzMask = (kCHS == 128) ? 7 : (kCHS == 64) ? 3 : 1;
  static constexpr int kMTiles = D / 16;                        // PV m-tiles (output dims)
  static constexpr int kWarps = 4;                              // consumer warps
  static constexpr int kThreads = (kWarps + 1) * 32;            // + one producer warp
  static constexpr int kRows = LP ? 4 : 8 * NT;                 // query rows per head
  // QK accumulator sets per n-tile: integer digits (LP: 2 x 2 digits; else 3),
  // FP8 parts (LP: hi|lo in one; else hi, lo)
  static constexpr int kAcc = kInt ? (LP ? 2 : 3) : (LP ? 1 : 2);
  static constexpr int kDigits = LP ? 4 : 3;
  static constexpr int kKSteps = kInt ? D / 32 : D / 16;
  static constexpr int kQWords = kKSteps * kAcc * 2;            // B-fragment words per lane
  static constexpr int kMaxSplits = 128;
  // Precomputed query fragments of one (sequence, KV head, row group) unit in
  // the workspace: NT x 32 lanes x kQWords words (lane-major), then the kRows
  // row logit multipliers, padded to 16 bytes.
  static constexpr int kUnitWords = (NT * 32 * kQWords + kRows + 3) / 4 * 4;
  // shared memory: the stage ring sized to the per-CTA budget (3 CTAs per SM with
  // one n-tile, 2 with two)
  static constexpr int kBudget = (NT == 1 ? 76800 : 115712) - 1024;
  static constexpr int kStagesRaw = kBudget / kStageBytes;
  static constexpr int kStages = kStagesRaw > 32 ? 32 : (kStagesRaw < 2 ? 2 : kStagesRaw);
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kBarOff = kRingBytes;
  // full, empty, item full/empty x2, fragments, and one that is never signalled
  // (the stall_consumers diagnostic)
  static constexpr int kNumBars = 2 * kStages + 6;
  static constexpr int kDescOff = kBarOff + kNumBars * 8;
  // the producer's item table: inclusive item prefix per sequence, for as many
  // sequences (a multiple of 32, at most 256) as the budget leaves room for
  static constexpr int kTableOff = kDescOff + 2 * 64;
  static constexpr int kTableRoom = (kBudget + 1024 - kTableOff) / 4;
  static constexpr int kTableSeqs = (kTableRoom >= 256 ? 256 : kTableRoom) / 32 * 32;
  static constexpr int kSmemBytes = kTableOff + kTableSeqs * 4;
  static_assert(kChunks % 2 == 0, "ldmatrix.x4 covers two 16-byte chunks");
  static_assert(kHeadTile % ((kSwzMask + 1) * 128) == 0, "tiles keep the swizzle-atom alignment");
  static_assert(kStages <= 32, "one producer lane per stage");
  static_assert(BS % kTok == 0, "whole stages per block");
  static_assert(kSmemBytes <= kBudget + 1024, "shared memory budget");
  static_assert(kTableSeqs >= 32, "item table holds at least one warp of sequences");
};

// One work item as published by the producer to the consumers (64 bytes).
struct ItemDesc {
  int valid;  // 0: no more work
  int b, hg, rg, split;
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

// First of the two adjacent output dims held by accumulator elements c0 / c2 of
// PV m-tile mt for a thread with group index g.
template <int KV>
__device__ __forceinline__ int out_dim(int mt, int g) {
  if constexpr (KV == PA_KV_INT4) return 32 * (mt >> 1) + 4 * g + 2 * (mt & 1);
  return 16 * mt + 2 * g;
}

// Head groups of the device.
__device__ __forceinline__ int head_groups(const FwdArgs& a) {
  return (a.Hk + kHeadsPerItem - 1) / kHeadsPerItem;
}

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
  return head_groups(a) * rg * ns;
}

// Rows, keys and block range of item `local` of sequence b.  Returns false (and
// leaves d.valid = 0) when the item has no keys (a causal row group that ends
// before this split starts).
template <int BS>
__device__ __forceinline__ bool decode_item(const FwdArgs& a, int rows_cta, int b, int local,
                                            int q0, int qb, int Lb, ItemDesc& d) {
  d.valid = 0;
  const int R = qb * a.G;  // rows of (b, head): row r = token r / G, head h * G + r % G
  const int rg_n = (R + rows_cta - 1) / rows_cta;
  int ns, bps;
  split_geometry((Lb + BS - 1) / BS, a.split_target, a.max_splits, &ns, &bps);
  d.split = local % ns;
  const int rest = local / ns;
  d.rg = rest % rg_n;
  d.hg = rest / rg_n;
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

// ---------------------------------------------------------------------------
// Query fragments of one head, built by one warp in registers.  Lane (g, tig)
// folds k_scale into the channels its B-operand words carry for B column g and
// encodes them; it also returns the logit multiplier C of that column's row:
//   integer caches: logit (log2 units) = C 2^-6 sum_d code_d q''_d, q'' digits
//   FP8           : logit = C sum_d code_d (hi_d + lo_d)
// with C = softmax_scale log2(e) 2^(e_kv + e_q).
// Word (s * kAcc + i) * 2 + r is b-register r of k-step s for accumulator set i;
// the channel of its byte / half e is
//   INT8: 32 s + 16 r + 4 tig + e     INT4: 32 s + 8 tig + 2 e + r
//   FP8 : 16 s + 4 tig + 2 r + e (e < 2)
// matching the channels ldmatrix hands the same thread for the K operand.
// B column g carries row g >> 1 (LP; digits / part g & 1) or row 8 nt + g.
// qh: the query of the sequence's first new token, query head h * G (global);
// row row0 + r of the (sequence, head) unit is token (row0 + r) / G, query head
// h * G + (row0 + r) % G; sks: k_scale row of head h.
template <int KV, int D, int BS, int NT, bool LP>
__device__ __forceinline__ void query_fragments(const FwdArgs& a, const uint8_t* qh,
                                                const float* sks, int row0, int nrows, int lane,
                                                uint32_t (&qf)[NT][Cfg<KV, D, BS, NT, LP>::kQWords],
                                                float (&crow)[NT]) {
  using C = Cfg<KV, D, BS, NT, LP>;
  const int g = lane >> 2, tig = lane & 3;
  // The thread's channels come in groups of kGS consecutive ones (INT4: 8, else
  // 4), so its query and scale values arrive in a few vector loads, all issued
  // before any arithmetic.  Group gi starts at channel
  //   INT8: 32 (gi >> 1) + 16 (gi & 1) + 4 tig   INT4: 32 gi + 8 tig   FP8: 16 gi + 4 tig
  // and its offset o is element 4 gi + o (INT8, FP8) or 8 gi + 4 (o & 1) + (o >> 1)
  // (INT4) of the list above.  The four lanes of one g cover every channel.
  constexpr int kN = D / 4;  // channels per lane
  constexpr int kGS = (KV == PA_KV_INT4) ? 8 : 4;
  constexpr int kNG = kN / kGS;
  auto gbase = [&](int gi) {
    if constexpr (KV == PA_KV_INT8) return 32 * (gi >> 1) + 16 * (gi & 1) + 4 * tig;
    else if constexpr (KV == PA_KV_INT4) return 32 * gi + 8 * tig;
    else return 16 * gi + 4 * tig;
  };
  auto elem = [](int gi, int o) {
    return (KV == PA_KV_INT4) ? 8 * gi + 4 * (o & 1) + (o >> 1) : 4 * gi + o;
  };
  float sc[kN];  // k_scale of element i's channel
#pragma unroll
  for (int gi = 0; gi < kNG; ++gi)
#pragma unroll
    for (int k = 0; k < kGS / 4; ++k) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(sks + gbase(gi) + 4 * k));
      sc[elem(gi, 4 * k + 0)] = v.x;
      sc[elem(gi, 4 * k + 1)] = v.y;
      sc[elem(gi, 4 * k + 2)] = v.z;
      sc[elem(gi, 4 * k + 3)] = v.w;
    }
  uint32_t qraw[NT][kN / 2];  // 16-bit query values of group gi at words gi kGS / 2 ..
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int row = LP ? (g >> 1) : nt * 8 + g;
    const int ru = row0 + row;
    const bool valid = row < nrows;
    const size_t roff = valid ? (static_cast<size_t>(ru / a.G) * a.H + ru % a.G) * D : 0;
    const uint16_t* qr = reinterpret_cast<const uint16_t*>(qh) + roff;
#pragma unroll
    for (int gi = 0; gi < kNG; ++gi) {
      if constexpr (kGS == 8) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (valid) v = __ldg(reinterpret_cast<const uint4*>(qr + gbase(gi)));
        qraw[nt][4 * gi + 0] = v.x;
        qraw[nt][4 * gi + 1] = v.y;
        qraw[nt][4 * gi + 2] = v.z;
        qraw[nt][4 * gi + 3] = v.w;
      } else {
        uint2 v = make_uint2(0u, 0u);
        if (valid) v = __ldg(reinterpret_cast<const uint2*>(qr + gbase(gi)));
        qraw[nt][2 * gi + 0] = v.x;
        qraw[nt][2 * gi + 1] = v.y;
      }
    }
  }
  float ksmax = 0.f;
  bool scale_ok = true;  // every K scale of the head finite (a NaN escapes fmaxf)
#pragma unroll
  for (int i = 0; i < kN; ++i) {
    ksmax = fmaxf(ksmax, fabsf(sc[i]));
    scale_ok &= isfinite(sc[i]);
  }
  ksmax = fmaxf(ksmax, __shfl_xor_sync(kFull, ksmax, 1));
  ksmax = fmaxf(ksmax, __shfl_xor_sync(kFull, ksmax, 2));
  if (__any_sync(kFull, !scale_ok) && lane == 0) record_error(a.err, PA_DEVERR_BAD_SCALE);
  int e_kv = 0;
  (void)frexpf(ksmax, &e_kv);
  const float f_kv = ldexpf(1.f, -e_kv);
  const bool qbf = a.q_bf16;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float w[kN];
    float rmax = 0.f;
#pragma unroll
    for (int gi = 0; gi < kNG; ++gi)
#pragma unroll
      for (int o = 0; o < kGS; ++o) {
        const uint32_t bits = (qraw[nt][gi * kGS / 2 + o / 2] >> (16 * (o & 1))) & 0xFFFFu;
        const float x = qbf ? __uint_as_float(bits << 16)
                            : __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
        const int i = elem(gi, o);
        w[i] = x * (sc[i] * f_kv);
        rmax = fmaxf(rmax, fabsf(w[i]));
      }
    rmax = fmaxf(rmax, __shfl_xor_sync(kFull, rmax, 1));
    rmax = fmaxf(rmax, __shfl_xor_sync(kFull, rmax, 2));
    int e_q = 0;
    (void)frexpf(rmax, &e_q);
    // The multiplier is capped at 2^90 (K scales or queries near FLT_MAX would
    // overflow it): the logits stay below 2^110, and two logits whose products
    // differ by 2^-31 of the query's digit unit or more still differ by >= 2^59
    // in log2 units, so the fp32 softmax weights are the same hard maximum the
    // uncapped values give.
    crow[nt] = fminf(ldexpf(a.sm_scale_log2, e_kv + e_q), 0x1p90f);
    if constexpr (C::kInt) {
      const float f = ldexpf(1.f, 6 - e_q);
      const int p = g & 1;
#pragma unroll
      for (int wd = 0; wd < kN / 4; ++wd) {  // word (s, r): elements 4 wd .. 4 wd + 3
        uint32_t dg[C::kDigits];
#pragma unroll
        for (int k = 0; k < C::kDigits; ++k) dg[k] = 0u;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v = w[4 * wd + e] * f;  // |v| < 64; each remainder times 128 stays within +-64
#pragma unroll
          for (int k = 0; k < C::kDigits; ++k) {
            const float t = rintf(v);
            dg[k] |= (static_cast<uint32_t>(static_cast<int>(t)) & 0xFFu) << (8 * e);
            v = (v - t) * 128.f;
          }
        }
        const int s = wd >> 1, r = wd & 1;
        if constexpr (LP) {
          // set i carries digit 2 i + p (p = g & 1)
          qf[nt][(s * 2 + 0) * 2 + r] = p ? dg[1] : dg[0];
          qf[nt][(s * 2 + 1) * 2 + r] = p ? dg[3] : dg[2];
        } else {
#pragma unroll
          for (int i = 0; i < 3; ++i) qf[nt][(s * 3 + i) * 2 + r] = dg[i];
        }
      }
    } else {
      const float f = ldexpf(1.f, -e_q);
#pragma unroll
      for (int wd = 0; wd < kN / 2; ++wd) {  // word (s, r): elements 2 wd, 2 wd + 1
        const float x0 = w[2 * wd] * f, x1 = w[2 * wd + 1] * f;  // |x| < 1
        const float h0 = __half2float(__float2half_rn(x0)), h1 = __half2float(__float2half_rn(x1));
        const uint32_t hi = pack_f32x2_to_h2(h0, h1);
        const uint32_t lo = pack_f32x2_to_h2(x0 - h0, x1 - h1);
        const int s = wd >> 1, r = wd & 1;
        if constexpr (LP) {
          qf[nt][s * 2 + r] = (g & 1) ? lo : hi;  // column g: part g & 1
        } else {
          qf[nt][(s * 2 + 0) * 2 + r] = hi;
          qf[nt][(s * 2 + 1) * 2 + r] = lo;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Fragment pre-pass: one warp per (sequence, KV head, row group) unit folds the
// K scale into the unit's query rows and stores every lane's B-operand words and
// the rows' logit multipliers in the workspace (query_fragments above), once per
// unit instead of once per split item.  The forward kernel is launched as this
// grid's programmatic dependent: it starts streaming KV right away and waits
// for this grid only before its consumers load fragments.  Two warps per CTA, so
// that a CTA fits beside three forward CTAs on one SM.
template <int KV, int D, int BS, int NT, bool LP>
__global__ void __launch_bounds__(64) pa_prep_kernel(const FwdArgs a) {
  using C = Cfg<KV, D, BS, NT, LP>;
  // This grid may be launched before the previous kernel of the stream has
  // finished (programmatic launch): nothing is read or written before that
  // grid's completion, and the forward kernel is released only after it.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  // unit (b, h, rg): the host keeps batch x Hk x row groups below 2^31
  const int units = a.batch * a.Hk * a.num_row_groups;
  const int u = blockIdx.x * 2 + (threadIdx.x >> 5);
  if (u >= units) return;
  const int bh = u / a.num_row_groups;
  const int rg = u - bh * a.num_row_groups;
  const int b = bh / a.Hk;
  const int h = bh - b * a.Hk;
  const int q0 = __ldg(a.cu_seqlens_q + b), qb = __ldg(a.cu_seqlens_q + b + 1) - q0;
  const int Lb = __ldg(a.seqlens_k + b);
  if (qb <= 0 || qb > Lb || q0 < 0 || q0 + qb > a.total_q) return;
  const int R = qb * a.G;
  const int row0 = rg * C::kRows;
  if (row0 >= R) return;
  const int nrows = min(R, row0 + C::kRows) - row0;
  uint32_t qf[NT][C::kQWords];
  float crow[NT];
  // the head's V scales must be finite too (checked once per sequence and head;
  // loaded first so that their latency overlaps the fold)
  float vsc[D / 32];
#pragma unroll
  for (int k = 0; k < D / 32; ++k)
    vsc[k] = rg == 0 ? __ldg(a.v_scale + static_cast<size_t>(h) * D + 32 * k + lane) : 0.f;
  const uint8_t* qh = reinterpret_cast<const uint8_t*>(a.q) +
                      (static_cast<size_t>(q0) * a.H + static_cast<size_t>(h) * a.G) * D * 2;
  query_fragments<KV, D, BS, NT, LP>(a, qh, a.k_scale + static_cast<size_t>(h) * D, row0, nrows,
                                     lane, qf, crow);
  bool v_ok = true;
#pragma unroll
  for (int k = 0; k < D / 32; ++k) v_ok &= isfinite(vsc[k]);
  if (__any_sync(kFull, !v_ok) && lane == 0) record_error(a.err, PA_DEVERR_BAD_SCALE);
  uint32_t* fb = a.frag + static_cast<size_t>(u) * C::kUnitWords;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int k4 = 0; k4 < C::kQWords / 4; ++k4)
      reinterpret_cast<uint4*>(fb + (nt * 32 + lane) * C::kQWords)[k4] =
          make_uint4(qf[nt][4 * k4], qf[nt][4 * k4 + 1], qf[nt][4 * k4 + 2], qf[nt][4 * k4 + 3]);
    // the lane of B column g holds the multiplier of row g >> 1 (LP) or 8 nt + g
    if (tig == 0 && (!LP || (g & 1) == 0))
      reinterpret_cast<float*>(fb + NT * 32 * C::kQWords)[LP ? (g >> 1) : nt * 8 + g] = crow[nt];
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

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  constexpr int rows_cta = C::kRows;

  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + C::kStages + s); };
  auto item_full = [&](int sl) { return smem_u32(bars + 2 * C::kStages + sl); };
  auto item_empty = [&](int sl) { return smem_u32(bars + 2 * C::kStages + 2 + sl); };
  // completes once every consumer warp holds its first item's query fragments
  const uint32_t frag_ready = smem_u32(bars + 2 * C::kStages + 4);
  // never completes: the consumers of a stall_consumers call wait on it
  const uint32_t never_bar = smem_u32(bars + 2 * C::kStages + 5);
  auto k_tile = [&](int s) { return smem + s * C::kStageBytes; };
  auto v_tile = [&](int s) { return smem + s * C::kStageBytes + C::kKTile; };

  // The combine kernel (launched after this one when the plan splits the KV)
  // may be scheduled onto SMs as this grid's CTAs finish; it waits for this
  // grid's completion before reading anything.
  asm volatile("griddepcontrol.launch_dependents;");
  // The producer's first global reads, the lengths of sequences 0..31 (lane b),
  // go out before the barrier set-up.
  const int nk = (a.batch + 31) >> 5;
  const bool dense = a.batch <= C::kTableSeqs;
  int f_q0 = 0, f_q1 = 0, f_L = 0;
  if (warp == C::kWarps && dense && lane < a.batch) {
    f_q0 = __ldg(a.cu_seqlens_q + lane);
    f_q1 = __ldg(a.cu_seqlens_q + lane + 1);
    f_L = __ldg(a.seqlens_k + lane);
  }
  if (warp == 0) {  // one barrier per lane
    for (int s = lane; s < C::kStages; s += 32) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), C::kWarps);
    }
    if (lane < 2) {
      mbar_init(item_full(lane), 1);
      mbar_init(item_empty(lane), C::kWarps);
    }
    if (lane == 2) mbar_init(frag_ready, C::kWarps);
    if (lane == 3) mbar_init(never_bar, 1);
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
    // ---- dense item numbering: per-sequence item counts and their prefix sums
    // in shared memory (compact rolled loops: this runs once per CTA on a cold
    // instruction cache); beyond kTableSeqs sequences the numbering is sparse
    // (every sequence gets the largest count; empty items are skipped).
    int* s_incl = reinterpret_cast<int*>(smem + C::kTableOff);
    int total = 0, per_seq = 0;
    if (dense) {
      bool bad_any = false;
#pragma unroll 1
      for (int k = 0; k < nk; ++k) {
        const int b = 32 * k + lane;
        int q0 = f_q0, q1 = f_q1, L = f_L;
        if (k > 0) {
          q0 = q1 = L = 0;
          if (b < a.batch) {
            q0 = __ldg(a.cu_seqlens_q + b);
            q1 = __ldg(a.cu_seqlens_q + b + 1);
            L = __ldg(a.seqlens_k + b);
          }
        }
        bool bad = false;
        int x = b < a.batch ? seq_items<BS>(a, rows_cta, q0, q1 - q0, L, bad) : 0;
        bad_any |= bad;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(kFull, x, o);
          if (lane >= o) x += y;
        }
        s_incl[b] = total + x;  // b < 32 nk <= kTableSeqs
        total += __shfl_sync(kFull, x, 31);
      }
      __syncwarp();
      if (bad_any) record_error(a.err, PA_DEVERR_BAD_LENGTH);
    } else {
      per_seq = head_groups(a) * a.num_row_groups * a.max_splits;
      total = a.batch * per_seq;
    }

    // Item w -> (sequence, index within the sequence, its lengths); false when
    // the item has no work.
    auto locate = [&](int w, ItemDesc& d) -> bool {
      d.valid = 0;
      if (dense) {
        // the first sequence whose inclusive prefix exceeds w
        int fb = -1;
#pragma unroll 1
        for (int k = 0; k < nk && fb < 0; ++k) {
          const int b = 32 * k + lane;
          const unsigned m = __ballot_sync(kFull, b < a.batch && s_incl[b] > w);
          if (m != 0u) fb = 32 * k + __ffs(m) - 1;
        }
        if (fb < 0) return false;
        const int base = fb > 0 ? s_incl[fb - 1] : 0;
        const int q0 = __ldg(a.cu_seqlens_q + fb);
        const int qb = __ldg(a.cu_seqlens_q + fb + 1) - q0;
        const int Lb = __ldg(a.seqlens_k + fb);
        return decode_item<BS>(a, rows_cta, fb, w - base, q0, qb, Lb, d);
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
      const int local = w - b * per_seq;
      // sparse layout: split fastest over max_splits, then row group, then head group
      const int split = local % a.max_splits;
      const int rest = local / a.max_splits;
      const int rg = rest % a.num_row_groups, hg = rest / a.num_row_groups;
      const int R = qb * a.G;
      const int rg_n = (R + rows_cta - 1) / rows_cta;
      int ns, bps;
      split_geometry((Lb + BS - 1) / BS, a.split_target, a.max_splits, &ns, &bps);
      if (rg >= rg_n || split >= ns) return false;
      return decode_item<BS>(a, rows_cta, b, (hg * rg_n + rg) * ns + split, q0, qb, Lb, d);
    };

    int uses0 = 0, uses1 = 0;  // items published in slot 0 / 1
    int fills = 0;             // copies issued into this lane's ring stage
    int slot = 0;
    int done = 0;  // stages issued so far: item stage kk lands in ring stage (done + kk) % kStages
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
      const int32_t* bt = a.block_table + static_cast<size_t>(d.b) * a.maxb + d.blk_begin;
      const int nst = d.valid ? d.nloc * C::kSPB : 0;
      // Lane l < kStages owns ring stage l and issues the item's stages kk with
      // (done + kk) % kStages == l, in order; first its block-table entry.
      const bool owner = lane < C::kStages;
      int kk = owner ? ((lane - done) % C::kStages + C::kStages) % C::kStages : 0;
      auto load_phys = [&](int kq) {
        int ph = __ldg(bt + kq / C::kSPB);
        if (ph < 0 || ph >= a.num_blocks) {
          record_error(a.err, PA_DEVERR_BAD_BLOCK);
          ph = a.num_blocks;  // out-of-range box: TMA fills zeros, nothing faults
        }
        return ph;
      };
      int phys = (owner && kk < nst) ? load_phys(kk) : 0;
      // publish the item (or the end marker) in the next slot
      if (lane == 0) {
        const int u = slot ? uses1 : uses0;
        if (u > 0 && !mbar_wait(item_empty(slot), (u - 1) & 1)) {
          record_error(a.err, PA_DEVERR_TIMEOUT);
          ok = false;
        } else {
          descs[slot] = d;
          mbar_arrive(item_full(slot));
        }
      }
      ok = __shfl_sync(kFull, ok, 0);
      if (slot) ++uses1; else ++uses0;
      if (!ok || !d.valid) break;

      // Each pass, every owner lane whose stage all four consumer warps have
      // released arms it and issues its two boxes (a non-blocking test, all lanes
      // in parallel), then fetches the block-table entry of its next stage; when
      // no lane could issue, one pending lane sleeps on its stage.
      // The CTA's first item: only two stages go out before the consumers hold
      // their query fragments, so that the fragment loads are not queued behind
      // the whole ring's worth of KV requests.
      bool gated = (done == 0);
      while (ok) {
        const bool pending = owner && kk < nst;
        const unsigned pend = __ballot_sync(kFull, pending);
        if (pend == 0u) break;
        bool issued = false;
        if (pending && !(gated && kk >= 2)) {
          const int round = (done + kk) / C::kStages;
          if (round == 0 || mbar_try_wait(empty_bar(lane), (round - 1) & 1)) {
            const int tok = phys * BS + (kk % C::kSPB) * C::kTok;
            const int hrow = d.hg * C::kHP;
            mbar_arrive_expect_tx(full_bar(lane), C::kStageBytes);
            tma_load_3d(smem_u32(k_tile(lane)), &kmap, full_bar(lane), 0, tok, hrow, policy);
            tma_load_3d(smem_u32(v_tile(lane)), &vmap, full_bar(lane), 0, tok, hrow, policy);
            ++fills;
            kk += C::kStages;
            if (kk < nst) phys = load_phys(kk);
            issued = true;
          }
        }
        if (__ballot_sync(kFull, issued) == 0u && gated) {
          if (lane == 0 && !mbar_wait(frag_ready, 0)) {
            record_error(a.err, PA_DEVERR_TIMEOUT);
            ok = false;
          }
          ok = __shfl_sync(kFull, ok, 0);
          gated = false;
        } else if (__ballot_sync(kFull, issued) == 0u) {
          // Nothing was free: sleep on the oldest pending stage.  Its release
          // needs no further issue (a consumer warp holds at most the two stages
          // before it), whereas a younger stage's release can wait on the very
          // stage this warp would then not be issuing.
          const unsigned key = pending ? static_cast<unsigned>(kk) : 0xFFFFFFFFu;
          const unsigned oldest = __reduce_min_sync(kFull, key);
          const int l0 = __ffs(__ballot_sync(kFull, pending && key == oldest)) - 1;
          if (lane == l0) {
            const int round = (done + kk) / C::kStages;
            if (!mbar_wait(empty_bar(lane), (round - 1) & 1)) {
              record_error(a.err, PA_DEVERR_TIMEOUT);
              ok = false;
            }
          }
          ok = __shfl_sync(kFull, ok, l0);
        }
      }
      if (done == 0) {
        // L2 prefetch of what later items and the epilogues read: the block
        // table and the V scale rows, strided over the CTAs
        auto prefetch_all = [&](const void* base, size_t bytes) {
          const size_t step = static_cast<size_t>(gridDim.x) * 32 * 128;
          for (size_t off = (static_cast<size_t>(blockIdx.x) * 32 + lane) * 128; off < bytes;
               off += step)
            prefetch_l2(reinterpret_cast<const uint8_t*>(base) + off);
        };
        prefetch_all(a.block_table, static_cast<size_t>(a.batch) * a.maxb * 4);
        prefetch_all(a.v_scale, static_cast<size_t>(a.Hk) * D * 4);
      }
      done += nst;
      slot ^= 1;
      w = next_index();
    }
    // The last prefetched index is consumed (its atomic has completed) before
    // this CTA signs off.
    const uint32_t last = __shfl_sync(kFull, w_pref, 0);
    // Leave no copy in flight: every owner lane waits for the last fill it
    // issued into its stage, all within one bounded window (the consumers
    // normally consumed them already).
    {
      const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
      const bool fine = fills == 0 || mbar_wait_until(full_bar(lane), (fills - 1) & 1, deadline);
      if (__ballot_sync(kFull, !fine) != 0u && lane == 0) record_error(a.err, PA_DEVERR_TIMEOUT);
    }
    if (lane == 0) {
      if (last == 0xffffffffu) record_error(a.err, PA_DEVERR_BAD_LENGTH);  // (never: uses the value)
      __threadfence();
      // The last CTA to finish rewinds the work counter for the next call.
      if (atomicAdd(a.work + 1, 1u) == gridDim.x - 1) {
        a.work[0] = 0u;
        a.work[1] = 0u;
      }
    }
    return;
  }

  // ======================================================== consumer warps
  int uses0 = 0, uses1 = 0;  // items taken from slot 0 / 1
  int slot = 0;
  bool prep_done = false;  // the fragment pre-pass grid has completed
  int kc = 0;  // stages consumed so far: item stage it is ring stage (kc + it) % kStages
  // ldmatrix lane addressing: matrix (lane >> 3) covers rows (lane & 7) + 8 * (m & 1)
  // of the 16-row head tile and chunk (2 cp + (m >> 1)).
  const int lm = lane >> 3;
  const int ld_row = (lane & 7) + 8 * (lm & 1);
  const int ld_chunk = lm >> 1;

  for (;;) {
    if (!__all_sync(kFull, mbar_wait(item_full(slot), (slot ? uses1 : uses0) & 1))) {
      if (lane == 0) record_error(a.err, PA_DEVERR_TIMEOUT);
      break;
    }
    if (slot) ++uses1; else ++uses0;
    const ItemDesc d = descs[slot];
    if (!d.valid) break;
    const int h = d.hg * C::kHP + warp;  // this warp's KV head
    const bool active = h < a.Hk;
    const int split = d.split, q0 = d.q0;
    const int row0 = d.row0, row_end = d.row_end, past = d.past, kmax = d.kmax, kfull = d.kfull;
    const int blk_begin = d.blk_begin, nloc = d.nloc, nsplit = d.nsplit, Lb = d.Lb;
    const int nrows = row_end - row0;
    const int nst = nloc * C::kSPB;

    // ---- prologue: this head's precomputed query fragments and row multipliers
    // (written by the pre-pass kernel, which this grid waits for once)
    const bool first_item = !prep_done;
    if (!prep_done) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      prep_done = true;
      // Diagnostic: a wait that nothing ends.  Its bound runs out, the warp
      // records the timeout and leaves; the producer's own bounded waits then
      // run out too and it drains every copy it issued before the CTA exits.
      if (a.stall_consumers && !mbar_wait(never_bar, 0)) {
        if (lane == 0) record_error(a.err, PA_DEVERR_TIMEOUT);
        return;
      }
    }
    uint32_t qf[NT][C::kQWords];
    float wA[NT][2], wB[NT][2];
    int lim[NT][2];
    {
      const uint32_t* fb =
          a.frag + (static_cast<size_t>(d.b) * a.Hk + (active ? h : 0)) * a.num_row_groups * C::kUnitWords +
          static_cast<size_t>(d.rg) * C::kUnitWords;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int k4 = 0; k4 < C::kQWords / 4; ++k4) {
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (active) v = __ldcg(reinterpret_cast<const uint4*>(fb + (nt * 32 + lane) * C::kQWords) + k4);
          qf[nt][4 * k4 + 0] = v.x;
          qf[nt][4 * k4 + 1] = v.y;
          qf[nt][4 * k4 + 2] = v.z;
          qf[nt][4 * k4 + 3] = v.w;
        }
      const float* crow = reinterpret_cast<const float*>(fb + NT * 32 * C::kQWords);
      // per accumulator column j: logit weights and causal limit (LP: j = 0 only,
      // the thread's row is tig)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int rl = LP ? tig : nt * 8 + 2 * tig + j;
          const float cr = active ? __ldcg(crow + rl) : 0.f;
          if constexpr (C::kInt) {
            const float base = cr * ((KV == PA_KV_INT4) ? (1.f / 131072.f) : (1.f / 8192.f));
            wA[nt][j] = base;                                                // C 2^-13 (/16 INT4)
            wB[nt][j] = LP ? base * (1.f / 16384.f) : base * (1.f / 128.f);  // digits 2|3 or 2
          } else {
            wA[nt][j] = cr;
            wB[nt][j] = 0.f;
          }
          lim[nt][j] = (row0 + rl < row_end && a.causal) ? past + (row0 + rl) / a.G : kmax - 1;
        }
    }

    if (first_item) {
      // the fragments are in registers (the empty asm consumes them), then the
      // producer may release the rest of the first item's stages
      asm volatile("" ::"r"(qf[0][0]), "r"(qf[0][C::kQWords - 1]), "f"(wA[0][0]), "f"(wA[NT - 1][1]));
      __syncwarp();
      if (lane == 0) mbar_arrive(frag_ready);
    }
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

    // Software-pipelined over stages: the QK products of stage it + 1 are issued
    // before the softmax and PV of stage it and read only in the next pass, so
    // their latency hides behind this stage's work.  Accumulator sets: integer
    // digits (int) or FP8 parts (float).
    using AccT = typename std::conditional<C::kInt, int, float>::type;
    AccT accC[C::kAcc][NT][4], accN[C::kAcc][NT][4];
    // QK products of ring stage s into acc (ldmatrix + MMA only).
    auto qk_issue = [&](int s, AccT (&acc)[C::kAcc][NT][4]) {
      const uint32_t kbase = smem_u32(k_tile(s) + warp * C::kHeadTile);
#pragma unroll
      for (int i = 0; i < C::kAcc; ++i)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[i][nt][e] = AccT(0);
#pragma unroll
      for (int cp = 0; cp < C::kChunks / 2; ++cp) {
        uint32_t r[4];
        const uint32_t off = ld_row * C::kCHS + (2 * cp + ld_chunk) * 16;
        ldsm_x4(kbase + swz<C::kSwzMask>(off), r);
        if constexpr (C::kInt) {
#pragma unroll
          for (int hh = 0; hh < (KV == PA_KV_INT4 ? 2 : 1); ++hh) {
            uint32_t a0, a1, a2, a3;
            int ks;
            if constexpr (KV == PA_KV_INT8) {
              a0 = r[0]; a1 = r[1]; a2 = r[2]; a3 = r[3];  // 32 channels, raw codes
              ks = cp;
            } else {
              // nibbles as signed bytes 16 x code: low nibbles shifted up, high masked
              const uint32_t x0 = r[2 * hh], x1 = r[2 * hh + 1];  // keys g, g+8; chunk 2cp+hh
              a0 = (x0 << 4) & 0xF0F0F0F0u;
              a1 = (x1 << 4) & 0xF0F0F0F0u;
              a2 = x0 & 0xF0F0F0F0u;
              a3 = x1 & 0xF0F0F0F0u;
              ks = 2 * cp + hh;
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int i = 0; i < C::kAcc; ++i)
                imma_16832<false>(acc[i][nt], a0, a1, a2, a3, qf[nt][(ks * C::kAcc + i) * 2],
                                  qf[nt][(ks * C::kAcc + i) * 2 + 1]);
          }
        } else {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int ks = 2 * cp + hh;  // 16-channel k-step
            uint32_t a0, a1, a2, a3;
            e4m3x4_to_h2x2(r[2 * hh], a0, a2);      // key g: channels +0,1 | +2,3
            e4m3x4_to_h2x2(r[2 * hh + 1], a1, a3);  // key g+8
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int i = 0; i < C::kAcc; ++i)
                mma_16816(acc[i][nt], a0, a1, a2, a3, qf[nt][(ks * C::kAcc + i) * 2],
                          qf[nt][(ks * C::kAcc + i) * 2 + 1]);
          }
        }
      }
    };
    // Raw logits (log2 units) of item stage it from its products, masked.
    // LP: X[0][eh] = key g + 8 eh of row tig.  Else X[nt][e]: key g + 8 (e >> 1),
    // row nt * 8 + 2 tig + (e & 1).
    auto qk_finish = [&](int it, const AccT (&acc)[C::kAcc][NT][4], float (&X)[NT][4]) {
      const int key0 = (blk_begin + it / C::kSPB) * BS + (it % C::kSPB) * C::kTok;
      const bool need_mask = key0 + 16 > kfull;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) X[nt][e] = 0.f;
      if constexpr (LP) {
#pragma unroll
        for (int eh = 0; eh < 2; ++eh) {
          float xv;
          if constexpr (C::kInt) {
            const int A = acc[0][0][2 * eh] * 128 + acc[0][0][2 * eh + 1];
            const int B2 = acc[1][0][2 * eh] * 128 + acc[1][0][2 * eh + 1];
            xv = fmaf(__int2float_rn(A), wA[0][0], __int2float_rn(B2) * wB[0][0]);
          } else {
            // columns 2 tig / 2 tig + 1: high part / residual of row tig
            xv = (float(acc[0][0][2 * eh]) + float(acc[0][0][2 * eh + 1])) * wA[0][0];
          }
          if (need_mask && key0 + g + 8 * eh > lim[0][0]) xv = -INFINITY;
          X[0][eh] = xv;
        }
      } else {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = e & 1;
            float xv;
            if constexpr (C::kInt) {
              const int A = acc[0][nt][e] * 128 + acc[1][nt][e];
              xv = fmaf(__int2float_rn(A), wA[nt][j], __int2float_rn(acc[2 % C::kAcc][nt][e]) * wB[nt][j]);
            } else {
              xv = (float(acc[0][nt][e]) + float(acc[1 % C::kAcc][nt][e])) * wA[nt][j];
            }
            if (need_mask && key0 + g + (e >> 1) * 8 > lim[nt][j]) xv = -INFINITY;
            X[nt][e] = xv;
          }
      }
    };
    // Two n-tiles, and FP8 with two parts per row, keep the stages sequential
    // (registers).
    constexpr bool kPipe = (NT == 1) && (C::kInt || LP);
    // A stage wait that gives up ends this warp (error flag set): it releases
    // nothing more, so no stage is refilled while a copy into it may be in flight.
    if (kPipe && nst > 0) {
      if (!__all_sync(kFull, mbar_wait(full_bar(kc % C::kStages), (kc / C::kStages) & 1))) {
        if (lane == 0) record_error(a.err, PA_DEVERR_TIMEOUT);
        return;
      }
      if (active) qk_issue(kc % C::kStages, accN);
    }
    for (int it = 0; it < nst; ++it) {
      const int s = (kc + it) % C::kStages;
      const bool has_next = it + 1 < nst;
      const int sn = (kc + it + 1) % C::kStages;
      const int sw = kPipe ? sn : s;  // the stage whose logits this pass computes
      if ((kPipe ? has_next : true) &&
          !__all_sync(kFull, mbar_wait(full_bar(sw), ((kc + it + (kPipe ? 1 : 0)) / C::kStages) & 1))) {
        if (lane == 0) record_error(a.err, PA_DEVERR_TIMEOUT);
        return;
      }
      if (active) {
        // this stage's logits from the products issued last pass, then the next
        // stage's products (the last pass reissues this stage's, unused); or,
        // unpipelined, this stage's products and logits
        float Xc[NT][4];
        if constexpr (kPipe) {
#pragma unroll
          for (int i = 0; i < C::kAcc; ++i)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) accC[i][nt][e] = accN[i][nt][e];
          qk_issue(has_next ? sn : s, accN);
        } else {
          qk_issue(s, accC);
        }
        qk_finish(it, accC, Xc);
        const uint32_t vbase = smem_u32(v_tile(s) + warp * C::kHeadTile);
        const int key0 = (blk_begin + it / C::kSPB) * BS + (it % C::kSPB) * C::kTok;

        // ---------------- online softmax with a lazily raised running max
        float X[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) X[nt][e] = Xc[nt][e] - msub[nt][LP ? 0 : (e & 1)];
        if constexpr (LP) {
          float mx = fmaxf(X[0][0], X[0][1]);
          if (__any_sync(kFull, mx > thr[0][0])) {
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
            if (mx > thr[0][0]) {
              const float mnew = mx + msub[0][0];
              const float alpha =
                  (m_run[0][0] == -INFINITY) ? 0.f : fast_exp2(m_run[0][0] - mnew);
#pragma unroll
              for (int mt = 0; mt < C::kMTiles; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) o[0][mt][e] *= alpha;
#pragma unroll
              for (int e = 0; e < 4; ++e) lacc[0][e] *= alpha;
              X[0][0] -= mx;
              X[0][1] -= mx;
              m_run[0][0] = mnew;
              msub[0][0] = mnew;
              thr[0][0] = 8.f;
            }
          }
          X[0][0] = fast_exp2(X[0][0]);  // <= 2^8: safe range for fp16
          X[0][1] = fast_exp2(X[0][1]);
        } else {
          float mx[NT][2];
          bool any = false;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              mx[nt][j] = fmaxf(X[nt][j], X[nt][j + 2]);
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
                  X[nt][j] -= m;
                  X[nt][j + 2] -= m;
                  m_run[nt][j] = mnew;
                  msub[nt][j] = mnew;
                  thr[nt][j] = 8.f;
                }
              }
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) X[nt][e] = fast_exp2(X[nt][e]);
        }

        // ---------------- O^T[dim, col] += V^T P^T
        uint32_t pb[NT][2];
        if constexpr (LP) {
          // (row tig; keys g, g+8) -> column n = g: b0 (keys 2tig, 2tig+1) and b1
          // (keys 2tig+8, 2tig+9) of row n / 2; movmatrix gives even lanes b0 and
          // odd lanes b1, the partner lane (lane ^ 4) the other.
          const uint32_t p = pack_f32x2_to_h2(X[0][0], X[0][1]);
          const uint32_t mtr = movmatrix_trans(p);
          const uint32_t y = __shfl_xor_sync(kFull, mtr, 4);
          pb[0][0] = (g & 1) ? y : mtr;
          pb[0][1] = (g & 1) ? mtr : y;
        } else {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            pb[nt][0] = movmatrix_trans(pack_f32x2_to_h2(X[nt][0], X[nt][1]));
            pb[nt][1] = movmatrix_trans(pack_f32x2_to_h2(X[nt][2], X[nt][3]));
          }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_16816(lacc[nt], kOnesH2, kOnesH2, kOnesH2, kOnesH2, pb[nt][0], pb[nt][1]);
#pragma unroll
        for (int cp = 0; cp < C::kChunks / 2; ++cp) {
          uint32_t r[4];
          const uint32_t off = ld_row * C::kCHS + (2 * cp + ld_chunk) * 16;
          ldsm_x4_trans(vbase + swz<C::kSwzMask>(off), r);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const uint32_t lo = r[2 * hf], hi = r[2 * hf + 1];  // keys 2tig.. / 2tig+8.. of chunk c
            const int c = 2 * cp + hf;
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
                if (key0 + 16 > Lb) {
                  // Keys past the sequence end hold stale bytes; an FP8 NaN there would
                  // poison P*V even with P = 0, so such V codes are zeroed.
                  const int kb = key0 + 2 * tig;
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
      if (lane == 0) mbar_arrive(empty_bar(s));
    }
    kc += nst;

    if (active) {
      // ---- remove the code->fp16 constants (using the exact row sums of P);
      // accumulator columns j (LP: both = row tig)
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

      // ---- normalise, apply the V scale, store the rows or the split partial
      const bool is_split = nsplit > 1;
      const float* vsc = a.v_scale + static_cast<size_t>(h) * D;
      const size_t stride = static_cast<size_t>(a.total_q) * a.H;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < (LP ? 1 : 2); ++j) {
          const int rl = LP ? tig : nt * 8 + 2 * tig + j;
          if (rl >= nrows) continue;
          const int r = row0 + rl;
          const size_t orow = static_cast<size_t>(q0 + r / a.G) * a.H + h * a.G + r % a.G;
          const float L = lacc[nt][LP ? 0 : j];
          const float inv = (L > 0.f) ? 1.f / L : 0.f;
          const size_t prow = static_cast<size_t>(split) * stride + orow;
#pragma unroll
          for (int mt = 0; mt < C::kMTiles; ++mt) {
            const int dd = out_dim<KV>(mt, g);
            if (!is_split) {
              const float2 vs = __ldg(reinterpret_cast<const float2*>(vsc + dd));
              const float o0 = o[nt][mt][j] * inv * vs.x;
              const float o1 = o[nt][mt][j + 2] * inv * vs.y;
              if (a.out_f32)
                *reinterpret_cast<float2*>(reinterpret_cast<float*>(a.out) + orow * D + dd) =
                    make_float2(o0, o1);
              else if (a.out_bf16)
                *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(a.out) +
                                                   orow * D + dd) = __floats2bfloat162_rn(o0, o1);
              else
                *reinterpret_cast<__half2*>(reinterpret_cast<__half*>(a.out) + orow * D + dd) =
                    __floats2half2_rn(o0, o1);
            } else {
              // the partial in code units (|o| <= max |code| <= 448): fp16 keeps
              // it within 2^-12 of its range; the combine applies the V scale
              *reinterpret_cast<__half2*>(a.o_part + prow * D + dd) =
                  __floats2half2_rn(o[nt][mt][j] * inv, o[nt][mt][j + 2] * inv);
            }
          }
          if (is_split && g == 0)
            a.lse_part[prow] = (L > 0.f) ? m_run[nt][j] + __log2f(L) : -INFINITY;
          // the row's log-sum-exp for callers that merge results (natural log)
          if (!is_split && a.lse_out != nullptr && g == 0)
            a.lse_out[orow] = (L > 0.f) ? (m_run[nt][j] + __log2f(L)) * 0.6931471805599453f
                                        : -INFINITY;
          // every row's split count, for the combine (1: stored above)
          if (a.row_ns != nullptr && split == 0 && g == 0) a.row_ns[orow] = nsplit;
        }

    }
    // the descriptor slot may be refilled
    __syncwarp();
    if (lane == 0) mbar_arrive(item_empty(slot));
    slot ^= 1;
  }
}

// ---------------------------------------------------------------------------
// Log-sum-exp merge of the split partials (flash decoding, GQA GEMV decode page,
// Code analysis 2: the workers' partials are combined after the split pass):
//   lse = log2 sum_s 2^lse_s,  out = sum_s 2^(lse_s - lse) o_s
// WPR warps per (new-token row, query head): four when the rows are few (one
// CTA per row; warp w takes splits w, w + 4, ...), else one (four rows per CTA).
// The forward kernel stored, for every row, how many splits of its (sequence,
// KV head, row group) have keys; rows of unsplit units (count 1) were stored by
// the forward kernel and are skipped.  Every load the merge needs goes out in
// one round trip after the wait: the count, the log-sum-exps of all planned
// splits and the partials of the warp's first splits; values of splits past
// the row's count are never used.  Launched as the forward kernel's
// programmatic dependent: it waits for the forward grid to complete before
// reading anything the forward grid wrote.
template <int D, int BS, int WPR>
__global__ void __launch_bounds__(128) pa_combine_kernel(const FwdArgs a) {
  __shared__ float4 red[3][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wsub = warp % WPR;                        // this warp's share of the splits
  const int gr = blockIdx.x * (4 / WPR) + warp / WPR;  // row of out viewed as [total_q * H]
  const bool row_ok = gr < a.total_q * a.H;
  const int hq = row_ok ? gr % a.H : 0;
  constexpr int kD4 = D / 4;  // lane handles dims 4 lane .. 4 lane + 3
  const bool dl = lane < kD4;
  const int P = a.max_splits;  // planned splits (partials allocated per split)
  // the V scale of the row's KV head (an input: read before the wait)
  float4 vs = make_float4(0.f, 0.f, 0.f, 0.f);
  if (row_ok && wsub == 0 && dl)
    vs = __ldg(reinterpret_cast<const float4*>(a.v_scale + static_cast<size_t>(hq / a.G) * D +
                                               4 * lane));
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the next call's pre-pass may be scheduled now (it waits for this grid)
  asm volatile("griddepcontrol.launch_dependents;");
  if (!row_ok) return;  // warp-uniform; a whole CTA when WPR = 4
  const size_t stride = static_cast<size_t>(a.total_q) * a.H;
  int S = __ldcg(a.row_ns + gr);
  float ls[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int sp = lane + 32 * k;
    ls[k] = sp < P ? __ldcg(a.lse_part + sp * stride + gr) : -INFINITY;
  }
  constexpr int kB = 8;  // partials in flight per lane
  const __half* base = a.o_part + static_cast<size_t>(gr) * D + 4 * (dl ? lane : 0);
  uint2 v[kB];
#pragma unroll
  for (int u = 0; u < kB; ++u) {
    const int sp = wsub + WPR * u;
    v[u] = (sp < P && dl) ? __ldcg(reinterpret_cast<const uint2*>(base + sp * stride * D))
                          : make_uint2(0u, 0u);
  }
  S = min(S, P);  // a row of an invalid sequence holds no count of this call
  if (S <= 1) return;  // uniform over the row's warps
  // weights 2^(lse_s - max) / sum over the row's splits
  float M = -INFINITY;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (lane + 32 * k >= S) ls[k] = -INFINITY;
    M = fmaxf(M, ls[k]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    ls[k] = (ls[k] == -INFINITY) ? 0.f : fast_exp2(ls[k] - M);
    sum += ls[k];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  if (a.lse_out != nullptr && wsub == 0 && lane == 0)  // merged log-sum-exp (natural log)
    a.lse_out[gr] = sum > 0.f ? (M + __log2f(sum)) * 0.6931471805599453f : -INFINITY;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int u0 = 0; wsub + WPR * u0 < S; u0 += kB) {
    if (u0 > 0) {  // splits beyond the first batch
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int sp = wsub + WPR * (u0 + u);
        v[u] = (sp < S && dl) ? __ldcg(reinterpret_cast<const uint2*>(base + sp * stride * D))
                              : make_uint2(0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int sp = wsub + WPR * (u0 + u);
      const float wv = __shfl_sync(kFull, ls[(sp >> 5) & 3], sp & 31) * inv;
      if (sp < S) {
        const float2 f01 = __half22float2(u2h2(v[u].x));
        const float2 f23 = __half22float2(u2h2(v[u].y));
        acc.x = fmaf(wv, f01.x, acc.x);
        acc.y = fmaf(wv, f01.y, acc.y);
        acc.z = fmaf(wv, f23.x, acc.z);
        acc.w = fmaf(wv, f23.y, acc.w);
      }
    }
  }
  if constexpr (WPR > 1) {  // the four warps' sums
    if (warp > 0) red[warp - 1][lane] = acc;
    __syncthreads();
    if (warp != 0) return;
#pragma unroll
    for (int w = 0; w < 3; ++w) {
      const float4 t = red[w][lane];
      acc.x += t.x;
      acc.y += t.y;
      acc.z += t.z;
      acc.w += t.w;
    }
  }
  if (!dl) return;
  acc.x *= vs.x;
  acc.y *= vs.y;
  acc.z *= vs.z;
  acc.w *= vs.w;
  const size_t o = static_cast<size_t>(gr) * D + 4 * lane;
  if (a.out_f32) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + o) = acc;
  } else if (a.out_bf16) {
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(a.out) + o);
    dst[0] = __floats2bfloat162_rn(acc.x, acc.y);
    dst[1] = __floats2bfloat162_rn(acc.z, acc.w);
  } else {
    __half2* dst = reinterpret_cast<__half2*>(reinterpret_cast<__half*>(a.out) + o);
    dst[0] = __floats2half2_rn(acc.x, acc.y);
    dst[1] = __floats2half2_rn(acc.z, acc.w);
  }
}

// Rows below this count get four warps each (one CTA per row).
constexpr long long kCombineSplitWarpRows = 1024;

template <int D, int BS>
static cudaError_t launch_combine_t(const FwdArgs& a, cudaStream_t stream) {
  const long long rows = static_cast<long long>(a.total_q) * a.H;
  if (rows <= 0) return cudaSuccess;
  // Like the forward kernels, the combine prefers the largest shared-memory
  // carveout, so that no SM is reconfigured between the kernels of a call.
  static std::atomic<int> configured[64] = {};
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return ce;
  if (dev >= 64 || !configured[dev].load(std::memory_order_acquire)) {
    ce = cudaFuncSetAttribute(pa_combine_kernel<D, BS, 1>, cudaFuncAttributePreferredSharedMemoryCarveout,
                              cudaSharedmemCarveoutMaxShared);
    if (ce != cudaSuccess) return ce;
    ce = cudaFuncSetAttribute(pa_combine_kernel<D, BS, 4>, cudaFuncAttributePreferredSharedMemoryCarveout,
                              cudaSharedmemCarveoutMaxShared);
    if (ce != cudaSuccess) return ce;
    if (dev < 64) configured[dev].store(1, std::memory_order_release);
  }
  const bool few = rows < kCombineSplitWarpRows;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(few ? rows : (rows + 3) / 4));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return few ? cudaLaunchKernelEx(&cfg, pa_combine_kernel<D, BS, 4>, a)
             : cudaLaunchKernelEx(&cfg, pa_combine_kernel<D, BS, 1>, a);
}

cudaError_t launch_combine(int head_size, int block_size, const FwdArgs& a, cudaStream_t stream) {
  if (head_size == 64 && block_size == 16) return launch_combine_t<64, 16>(a, stream);
  if (head_size == 64 && block_size == 32) return launch_combine_t<64, 32>(a, stream);
  if (head_size == 128 && block_size == 16) return launch_combine_t<128, 16>(a, stream);
  if (head_size == 128 && block_size == 32) return launch_combine_t<128, 32>(a, stream);
  return cudaErrorInvalidValue;
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
    // All three kernels of a call prefer the largest shared-memory carveout, so
    // an SM that ran a pre-pass or combine CTA need not be reconfigured before
    // it can take forward CTAs.
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(pa_prep_kernel<KV, D, BS, NT, LP>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(pa_combine_kernel<D, BS, 1>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(pa_combine_kernel<D, BS, 4>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, C::kThreads, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    if (dev < 64) ctas_per_sm[dev].store(per_sm, std::memory_order_release);
  }
  const long long slots = static_cast<long long>(per_sm) * a.num_sms;
  const int grid = static_cast<int>(a.num_items < slots ? a.num_items : slots);
  if (grid < 1) return cudaSuccess;
  // the fragment pre-pass, then the forward kernel as its programmatic dependent
  // the fragment pre-pass (a programmatic dependent of whatever precedes it in
  // the stream: it waits for that grid before touching memory)
  const long long units = static_cast<long long>(a.batch) * a.Hk * a.num_row_groups;
  if (units >= (1ll << 31)) return cudaErrorInvalidValue;
  {
    cudaLaunchConfig_t pc = {};
    pc.gridDim = dim3(static_cast<unsigned>((units + 1) / 2));
    pc.blockDim = dim3(64);
    pc.stream = stream;
    cudaLaunchAttribute pattr[1];
    pattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pattr[0].val.programmaticStreamSerializationAllowed = 1;
    pc.attrs = pattr;
    pc.numAttrs = 1;
    e = cudaLaunchKernelEx(&pc, pa_prep_kernel<KV, D, BS, NT, LP>, a);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, kmap, vmap, a);
}

template <int KV, int D, int BS, int NT, bool LP>
static int smem_t() {
  return Cfg<KV, D, BS, NT, LP>::kSmemBytes;
}

template <int KV, int D>
static int unit_words_t(int rows) {
  if (rows == 4) return Cfg<KV, D, 16, 1, true>::kUnitWords;
  if (rows == 8) return Cfg<KV, D, 16, 1, false>::kUnitWords;
  if (rows == 16) return Cfg<KV, D, 16, 2, false>::kUnitWords;
  return -1;
}

int fragment_unit_words(int kv_dtype, int head_size, int rows_per_cta) {
  if (rows_per_cta == prefill_rows_per_item()) return prefill_unit_words();
  const bool d128 = head_size == 128;
  switch (kv_dtype) {
    case PA_KV_INT8:
      return d128 ? unit_words_t<PA_KV_INT8, 128>(rows_per_cta)
                  : unit_words_t<PA_KV_INT8, 64>(rows_per_cta);
    case PA_KV_INT4:
      return d128 ? unit_words_t<PA_KV_INT4, 128>(rows_per_cta)
                  : unit_words_t<PA_KV_INT4, 64>(rows_per_cta);
    case PA_KV_FP8_E4M3:
      return d128 ? unit_words_t<PA_KV_FP8_E4M3, 128>(rows_per_cta)
                  : unit_words_t<PA_KV_FP8_E4M3, 64>(rows_per_cta);
    default:
      return -1;
  }
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
