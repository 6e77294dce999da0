// pa_attention.cu -- fused paged quantised-KV GQA attention for sm_100a.
//
// One CTA owns one (KV head, group of query rows, sequence, KV split).  Its rows
// are (new token, query head of the group) pairs of one sequence, so every row
// reads the same keys: the GQA group x new tokens form the N side of a
// tensor-core tile, keys form the M side ("swap-AB"), channels the K side.
//
// Data path:
//   producer warp : bulk copies of the CTA's query rows and both per-channel
//                   scale rows into shared memory, then, per KV block,
//                   block_table -> two 3-D TMA boxes (K rows, V rows of one
//                   head) into a swizzled stage of an mbarrier ring.
//   consumer warps: fold the K scale into the queries (fp16 high part plus fp16
//                   residual), then per 32 keys: ldmatrix (K) -> exact
//                   code->fp16 conversion in registers -> mma.sync m16n8k16 with
//                   fp32 accumulators -> online softmax in the exp2 domain whose
//                   running maximum is only raised (shuffle reduction and
//                   rescale) when a logit exceeds it by more than 2^8 ->
//                   P^T to fp16 with movmatrix -> ldmatrix.trans (V) ->
//                   conversion -> mma.sync into O^T.
// The four consumer warps take alternate 32-key groups and merge (m, l, O)
// through shared memory at the end, where the per-channel V scale is applied
// once.  With num_splits > 1 each CTA writes a normalised partial and its
// log2-sum-exp; the last CTA of a (sequence, KV head, row group) to finish,
// found with an arrival counter in the workspace, merges the splits and resets
// the counter.
//
// Sources: the per-channel K scale folded into Q with a power-of-two normaliser
// (INT4 paged-KV page, onnxruntime PR 32515, Code analysis 3); INT8 codes kept
// raw and converted to FP16 in registers right before an m16n8k16 MMA with FP32
// accumulation (INT8-KV tensor-core page, onnxruntime PR 33707, Code analysis
// 1); online softmax, masking and the flash-decoding split with a partials
// buffer (GQA GEMV decode page, onnxruntime PR 29216, Code analysis 1-2); the
// grid sized by the exact max_query_len (exact max_query_len page, onnxruntime
// PR 28409, Code analysis 2).
#include <math.h>

#include <atomic>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// NT: 8-row n-tiles per CTA (rows = 8 NT).  LOPACK (NT = 1 only): the CTA has at
// most 4 rows; B-operand columns 0..3 carry the fp16 high parts of the folded
// queries and columns 4..7 their residuals, so one MMA per k-step gives both.
template <int KV, int D, int BS, int NT, bool LOPACK>
struct Cfg {
  static constexpr int kCHS = (KV == PA_KV_INT4) ? D / 2 : D;  // cache bytes per row
  static constexpr int kTile = BS * kCHS;                       // one block, one head
  static constexpr int kStageBytes = 2 * kTile;                 // K + V
  static constexpr int kChunks = kCHS / 16;                     // 16-byte chunks per row
  static constexpr int kSwzMask = (kCHS == 128) ? 7 : (kCHS == 64) ? 3 : 1;
  static constexpr int kKSteps = D / 16;                        // QK k-steps
  static constexpr int kMTiles = D / 16;                        // PV m-tiles (output dims)
  static constexpr int kKeyTiles = BS / 16;                     // 16-key tiles per block
  static constexpr int kBPI = (BS == 16) ? 2 : 1;               // blocks per warp iteration
  static constexpr int kTPI = kBPI * kKeyTiles;                 // key tiles per iteration (2)
  static constexpr int kWarps = 4;                              // consumer warps
  static constexpr int kThreads = (kWarps + 1) * 32;            // + one producer warp
  static constexpr int kStageUnit = kWarps * kBPI;
  static constexpr int kStagesRaw = 32768 / kStageBytes;
  static constexpr int kStages = kStagesRaw < 2 * kStageUnit
                                     ? 2 * kStageUnit
                                     : ((kStagesRaw + kStageUnit - 1) / kStageUnit) * kStageUnit;
  static constexpr int kRows = 8 * NT;
  static constexpr int kQF = LOPACK ? 2 : 4;                    // query registers per k-step
  static constexpr int kPipeBytes = kStages * kStageBytes;
  static constexpr int kEpiBytes = kWarps * kRows * D * 4;
  static constexpr int kDataBytes = kPipeBytes > kEpiBytes ? kPipeBytes : kEpiBytes;
  static constexpr int kQOff = kDataBytes;                      // query rows (fp16 / bf16)
  static constexpr int kKsOff = kQOff + kRows * D * 2;          // k_scale row (fp32)
  static constexpr int kVsOff = kKsOff + D * 4;                 // v_scale row (fp32)
  static constexpr int kBarOff = kVsOff + D * 4;                // full[S], empty[S], qbar
  static constexpr int kStatOff = kBarOff + (2 * kStages + 2) * 8;
  static constexpr int kFlagOff = kStatOff + 2 * kWarps * kRows * 4;
  static constexpr int kSmemBytes = 1024 + kFlagOff + 16;
  static_assert(kChunks % 2 == 0, "ldmatrix.x4 covers two 16-byte chunks");
  static_assert(kStages % kStageUnit == 0, "stages are owned by one consumer warp each");
  static_assert(kTile % ((kSwzMask + 1) * 128) == 0, "tiles keep the swizzle-atom alignment");
  static_assert(!LOPACK || NT == 1, "residual packing needs a single n-tile");
  static_assert(kTPI == 2, "two 16-key tiles per warp iteration");
};

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

// Channel of the query operand for QK k-step s, half j (j = 0,1 -> first B
// register, 2,3 -> second), for the thread with index tig in its quad.  It
// matches the channels that ldmatrix hands the same thread for the K operand.
template <int KV>
__device__ __forceinline__ int q_channel(int s, int j, int tig) {
  if constexpr (KV == PA_KV_INT4) {
    constexpr int kOff[4] = {0, 4, 1, 5};
    return 32 * (s >> 1) + 8 * tig + 2 * (s & 1) + kOff[j];
  } else {
    return 16 * s + 4 * tig + j;
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

template <int KV, int D, int BS, int NT, bool LOPACK>
__global__ void __launch_bounds__(Cfg<KV, D, BS, NT, LOPACK>::kThreads)
    pa_fwd_kernel(const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap, const FwdArgs a) {
  using C = Cfg<KV, D, BS, NT, LOPACK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);  // full | empty | qbar
  float* sm_m = reinterpret_cast<float*>(smem + C::kStatOff);
  float* sm_l = sm_m + C::kWarps * C::kRows;
  int* sm_flag = reinterpret_cast<int*>(smem + C::kFlagOff);
  float* epi = reinterpret_cast<float*>(smem);  // aliases the stages after the loop
  const float* sks = reinterpret_cast<const float*>(smem + C::kKsOff);
  const float* svs = reinterpret_cast<const float*>(smem + C::kVsOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;

  const int rg = blockIdx.x % a.num_row_groups;
  const int kv = blockIdx.x / a.num_row_groups;
  const int b = blockIdx.y;
  const int split = blockIdx.z;

  // ---- this CTA's rows and keys (device copies of the lengths)
  const int q0 = a.cu_seqlens_q[b];
  const int qb = a.cu_seqlens_q[b + 1] - q0;
  const int Lb = a.seqlens_k[b];
  if (q0 < 0 || qb < 0 || qb > Lb || q0 + qb > a.total_q ||
      static_cast<long long>(Lb) > static_cast<long long>(a.maxb) * BS) {
    if (threadIdx.x == 0) record_error(a.err, PA_DEVERR_BAD_LENGTH);
    return;
  }
  const int R = qb * a.G;  // rows of (b, kv): row r = token (r / G), head kv*G + r % G
  const int rows_cta = LOPACK ? 4 : C::kRows;
  const int row0 = rg * rows_cta;
  if (row0 >= R) return;  // zero new tokens, or fewer rows than this row group
  const int row_end = min(R, row0 + rows_cta);
  const int past = Lb - qb;
  const int i_first = row0 / a.G;
  const int i_last = (row_end - 1) / a.G;
  const int kmax = a.causal ? past + i_last + 1 : Lb;    // keys seen by some row
  const int kfull = a.causal ? past + i_first + 1 : Lb;  // keys seen by every row
  const int nblk = (kmax + BS - 1) / BS;
  const int blk_begin = split * a.blocks_per_split;
  const int blk_end = min(nblk, blk_begin + a.blocks_per_split);
  const int nloc = max(0, blk_end - blk_begin);

  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + C::kStages + s); };
  const uint32_t qbar = smem_u32(bars + 2 * C::kStages);
  auto k_tile = [&](int s) { return smem + s * C::kStageBytes; };
  auto v_tile = [&](int s) { return smem + s * C::kStageBytes + C::kTile; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(qbar, 1);
    mbar_fence_init();
  }
  __syncthreads();

  // ======================================================== producer warp
  if (warp == C::kWarps) {
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      // Query rows of this CTA (contiguous per token) and both scale rows first.
      const uint32_t row_bytes = D * 2;
      const uint32_t total = static_cast<uint32_t>(row_end - row0) * row_bytes + 2 * D * 4;
      mbar_arrive_expect_tx(qbar, total);
      for (int i = i_first; i <= i_last; ++i) {
        const int r_lo = max(row0, i * a.G), r_hi = min(row_end, (i + 1) * a.G);
        const uint8_t* src =
            reinterpret_cast<const uint8_t*>(a.q) +
            ((static_cast<size_t>(q0 + i) * a.H + kv * a.G + (r_lo - i * a.G)) * D) * 2;
        bulk_load(smem_u32(smem + C::kQOff + (r_lo - row0) * row_bytes), src,
                  static_cast<uint32_t>(r_hi - r_lo) * row_bytes, qbar);
      }
      bulk_load(smem_u32(smem + C::kKsOff), a.k_scale + kv * D, D * 4, qbar);
      bulk_load(smem_u32(smem + C::kVsOff), a.v_scale + kv * D, D * 4, qbar);
    }
    if (nloc == 0) {
      if (lane == 0 && !mbar_wait(qbar, 0)) record_error(a.err, PA_DEVERR_TIMEOUT);
      return;
    }
    const uint64_t policy = l2_evict_first_policy();
    const int32_t* bt = a.block_table + static_cast<size_t>(b) * a.maxb + blk_begin;
    // Blocks go out in groups of kGroup (<= kStages, so every block of a group has
    // its own stage): lane j of the warp waits for its stage to be released,
    // arms it and issues the two boxes, all lanes in parallel.
    constexpr int kGroup = C::kStages < 32 ? C::kStages : 32;
    bool ok = true;
    int issued = 0;
    for (int base = 0; base < nloc; base += kGroup) {
      const int lb = base + lane;
      bool mine_ok = true;
      if (lane < kGroup && lb < nloc) {
        int phys = __ldg(bt + lb);
        if (phys < 0 || phys >= a.num_blocks) {
          record_error(a.err, PA_DEVERR_BAD_BLOCK);
          phys = a.num_blocks;  // out-of-range box: TMA fills zeros, nothing faults
        }
        const int s = lb % C::kStages;
        const int round = lb / C::kStages;
        if (round > 0 && !mbar_wait(empty_bar(s), (round - 1) & 1)) {
          mine_ok = false;
        } else {
          mbar_arrive_expect_tx(full_bar(s), C::kStageBytes);
          tma_load_3d(smem_u32(k_tile(s)), &kmap, full_bar(s), 0, kv, phys * BS, policy);
          tma_load_3d(smem_u32(v_tile(s)), &vmap, full_bar(s), 0, kv, phys * BS, policy);
        }
      }
      issued = min(nloc, base + kGroup);  // the drain below covers a partial group too
      ok = __all_sync(0xffffffffu, mine_ok);
      if (!ok) {
        if (lane == 0) record_error(a.err, PA_DEVERR_TIMEOUT);
        break;
      }
    }
    // Leave no copy in flight: wait for the last box of every stage and for the
    // query copies, all within one bounded window.
    if (lane == 0) {
      const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
      bool fine = mbar_wait_until(qbar, 0, deadline);
      for (int s = 0; fine && s < C::kStages && s < issued; ++s) {
        const int last_round = (issued - 1 - s) / C::kStages;
        fine = mbar_wait_until(full_bar(s), last_round & 1, deadline);
      }
      if (!fine) record_error(a.err, PA_DEVERR_TIMEOUT);
    }
    (void)ok;
    return;
  }

  // ======================================================== consumer warps
  bool alive = mbar_wait(qbar, 0);
  if (!alive && lane == 0) record_error(a.err, PA_DEVERR_TIMEOUT);

  // ---- prologue: fold the K scale into the queries.  q'[d] = q[d] k_scale[d] /
  // 2^e_kv (2^e_kv: power of two of max |k_scale| of this head), then a second
  // power of two per row keeps |q'| < 1 for any finite input before rounding to
  // fp16; both powers move into the per-row logit multiplier c (exp2 domain).
  float ksmax = 0.f;
#pragma unroll
  for (int d = lane; d < D; d += 32) ksmax = fmaxf(ksmax, fabsf(sks[d]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ksmax = fmaxf(ksmax, __shfl_xor_sync(0xffffffffu, ksmax, o));
  if (!isfinite(ksmax) && warp == 0 && lane == 0) record_error(a.err, PA_DEVERR_BAD_SCALE);
  int e_kv = 0;
  (void)frexpf(ksmax, &e_kv);
  const float f_kv = ldexpf(1.f, -e_kv);

  // qf[nt][s][0..1]: fp16 high parts of q' for k-step s; [2..3] (or, with LOPACK,
  // columns 4..7 of [0..1]): the fp16 rounding residuals q' - hi.  Together
  // they give the logits ~22 significant bits of q', enough when large
  // per-channel scales push logits into the hundreds.
  uint32_t qf[NT][C::kKSteps][C::kQF];
  float crow[NT][2];
  int lim[NT][2];
  const __half* sq16 = reinterpret_cast<const __half*>(smem + C::kQOff);
  const __nv_bfloat16* sqbf = reinterpret_cast<const __nv_bfloat16*>(smem + C::kQOff);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int rl = LOPACK ? (g & 3) : nt * 8 + g;  // local row of B-operand column g
    const bool valid = row0 + rl < row_end;
    float w[C::kKSteps][4];
    float rmax = 0.f;
#pragma unroll
    for (int s = 0; s < C::kKSteps; ++s) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int ch = q_channel<KV>(s, j, tig);
        float x = 0.f;
        if (valid)
          x = a.q_bf16 ? __bfloat162float(sqbf[rl * D + ch]) : __half2float(sq16[rl * D + ch]);
        w[s][j] = x * (sks[ch] * f_kv);
        rmax = fmaxf(rmax, fabsf(w[s][j]));
      }
    }
    rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 1));
    rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 2));
    int e_q = 0;
    (void)frexpf(rmax, &e_q);
    const float f_q = ldexpf(1.f, -e_q);
#pragma unroll
    for (int s = 0; s < C::kKSteps; ++s) {
      float hi[4], lo[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float xn = w[s][j] * f_q;
        hi[j] = __half2float(__float2half_rn(xn));
        lo[j] = xn - hi[j];
      }
      if constexpr (LOPACK) {
        const bool use_lo = g >= 4;
        qf[nt][s][0] = pack_f32x2_to_h2(use_lo ? lo[0] : hi[0], use_lo ? lo[1] : hi[1]);
        qf[nt][s][1] = pack_f32x2_to_h2(use_lo ? lo[2] : hi[2], use_lo ? lo[3] : hi[3]);
      } else {
        qf[nt][s][0] = pack_f32x2_to_h2(hi[0], hi[1]);
        qf[nt][s][1] = pack_f32x2_to_h2(hi[2], hi[3]);
        qf[nt][s][2] = pack_f32x2_to_h2(lo[0], lo[1]);
        qf[nt][s][3] = pack_f32x2_to_h2(lo[2], lo[3]);
      }
    }
    const float c_mine = ldexpf(a.sm_scale_log2, e_kv + e_q);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      // local row of accumulator column 2 tig + j
      const int rr = LOPACK ? ((2 * tig + j) & 3) : nt * 8 + 2 * tig + j;
      crow[nt][j] = __shfl_sync(0xffffffffu, c_mine, (LOPACK ? rr : (rr - nt * 8)) * 4);
      lim[nt][j] = (row0 + rr < row_end && a.causal) ? past + (row0 + rr) / a.G : kmax - 1;
    }
  }

  float o[NT][C::kMTiles][4];
  float m_run[NT][2], l_run[NT][2];
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
      const int lb = lb0 + bi;
      if (!mbar_wait(full_bar(lb % C::kStages), (lb / C::kStages) & 1)) {
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
      const uint32_t kbase = smem_u32(k_tile((lb0 + bi) % C::kStages));
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
          const uint32_t x0 = r[2 * h], x1 = r[2 * h + 1];  // rows g, g+8 of chunk 2cp+h
          const int c = 2 * cp + h;
#pragma unroll
          for (int hh = 0; hh < (KV == PA_KV_INT4 ? 2 : 1); ++hh) {
            uint32_t a0, a1, a2, a3;
            int ks;
            if constexpr (KV == PA_KV_INT8) {
              const uint32_t y0 = x0 ^ 0x80808080u, y1 = x1 ^ 0x80808080u;
              a0 = i8x2_to_h2(y0, 0x4140);
              a1 = i8x2_to_h2(y1, 0x4140);
              a2 = i8x2_to_h2(y0, 0x4342);
              a3 = i8x2_to_h2(y1, 0x4342);
              ks = c;
            } else if constexpr (KV == PA_KV_FP8_E4M3) {
              a0 = e4m3x2_to_h2(x0);
              a1 = e4m3x2_to_h2(x1);
              a2 = e4m3x2_to_h2(x0 >> 16);
              a3 = e4m3x2_to_h2(x1 >> 16);
              ks = c;
            } else {  // INT4: one 16-byte chunk = 32 channels = two k-steps
              const uint32_t z0 = x0 >> (8 * hh), z1 = x1 >> (8 * hh);
              a0 = i4lo_to_h2(z0);
              a1 = i4lo_to_h2(z1);
              a2 = i4hi_to_h2(z0);
              a3 = i4hi_to_h2(z1);
              ks = 2 * c + hh;
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              mma_16816(sacc[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
              if constexpr (!LOPACK)
                mma_16816(sres[nt], a0, a1, a2, a3, qf[nt][ks][2], qf[nt][ks][3]);
            }
          }
        }
      }
      const int key0 = (blk_begin + lb0 + bi) * BS + kt * 16;
      const bool need_mask = key0 + 16 > kfull;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float sv = sacc[nt][e];
          if constexpr (LOPACK)
            sv += __shfl_xor_sync(0xffffffffu, sv, 2);  // high part + residual part
          else
            sv += sres[nt][e];
          float xv = sv * crow[nt][e & 1];
          if (need_mask && key0 + g + (e >> 1) * 8 > lim[nt][e & 1]) xv = -INFINITY;
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
          const float p0 = fast_exp2(x[t][nt][j] - m_ref);  // <= 2^8: safe range for fp16
          const float p1 = fast_exp2(x[t][nt][j + 2] - m_ref);
          x[t][nt][j] = p0;
          x[t][nt][j + 2] = p1;
          l_run[nt][j] += p0 + p1;
        }
      }
    }

    // ---------------- O^T[dim, row] += V^T P^T, per key tile
#pragma unroll
    for (int t = 0; t < C::kTPI; ++t) {
      if (t >= ntiles) continue;
      const int bi = t / C::kKeyTiles, kt = t % C::kKeyTiles;
      const uint32_t vbase = smem_u32(v_tile((lb0 + bi) % C::kStages));
      // P^T as the B operand: (key g; rows 2tig, 2tig+1) -> (keys 2tig, 2tig+1; row g)
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        pb[nt][0] = movmatrix_trans(pack_f32x2_to_h2(x[t][nt][0], x[t][nt][1]));
        pb[nt][1] = movmatrix_trans(pack_f32x2_to_h2(x[t][nt][2], x[t][nt][3]));
      }
      // Keys past the sequence end in the last block hold stale bytes; an FP8 NaN
      // there would poison P*V even with P = 0, so such V codes are zeroed.
      uint32_t vmask_lo = 0xffffffffu, vmask_hi = 0xffffffffu;
      if constexpr (KV == PA_KV_FP8_E4M3) {
        const int kb = (blk_begin + lb0 + bi) * BS + kt * 16 + 2 * tig;
        if (kb + 9 >= Lb) {
          vmask_lo = (kb < Lb ? 0x0000ffffu : 0u) | (kb + 1 < Lb ? 0xffff0000u : 0u);
          vmask_hi = (kb + 8 < Lb ? 0x0000ffffu : 0u) | (kb + 9 < Lb ? 0xffff0000u : 0u);
        }
      }
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
              const uint32_t ylo = lo ^ 0x80808080u, yhi = hi ^ 0x80808080u;
              a0 = i8x2_to_h2(ylo, 0x4240);
              a1 = i8x2_to_h2(ylo, 0x4341);
              a2 = i8x2_to_h2(yhi, 0x4240);
              a3 = i8x2_to_h2(yhi, 0x4341);
              mt = c;
            } else if constexpr (KV == PA_KV_FP8_E4M3) {
              const uint32_t zlo = prmt(lo, 0u, 0x3120), zhi = prmt(hi, 0u, 0x3120);
              a0 = e4m3x2_to_h2(zlo) & vmask_lo;
              a1 = e4m3x2_to_h2(zlo >> 16) & vmask_lo;
              a2 = e4m3x2_to_h2(zhi) & vmask_hi;
              a3 = e4m3x2_to_h2(zhi >> 16) & vmask_hi;
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
      for (int bi = 0; bi < nb; ++bi) mbar_arrive(empty_bar((lb0 + bi) % C::kStages));
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
  consumer_sync();  // every warp left the pipeline: the stages may be reused
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int row = nt * 8 + 2 * tig + j;
      if (!writer) continue;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < C::kWarps; ++w) M = fmaxf(M, sm_m[w * C::kRows + row]);
      const float f = (m_run[nt][j] == -INFINITY) ? 0.f : fast_exp2(m_run[nt][j] - M);
#pragma unroll
      for (int mt = 0; mt < C::kMTiles; ++mt) {
        const int d = out_dim<KV>(mt, g);
        *reinterpret_cast<float2*>(epi + (warp * C::kRows + row) * D + d) =
            make_float2(o[nt][mt][j] * f, o[nt][mt][j + 2] * f);
      }
    }
  consumer_sync();

  const int nthr = C::kWarps * 32;
  const int nrows = row_end - row0;
  for (int idx = threadIdx.x; idx < nrows * (D / 2); idx += nthr) {
    const int row = idx / (D / 2);
    const int d = (idx % (D / 2)) * 2;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < C::kWarps; ++w) M = fmaxf(M, sm_m[w * C::kRows + row]);
    float L = 0.f, s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int w = 0; w < C::kWarps; ++w) {
      const float mw = sm_m[w * C::kRows + row];
      if (mw != -INFINITY) L += sm_l[w * C::kRows + row] * fast_exp2(mw - M);
      const float2 v = *reinterpret_cast<const float2*>(epi + (w * C::kRows + row) * D + d);
      s0 += v.x;
      s1 += v.y;
    }
    const float inv = (L > 0.f) ? 1.f / L : 0.f;
    const float o0 = s0 * inv * svs[d];
    const float o1 = s1 * inv * svs[d + 1];
    const int r = row0 + row;
    const size_t orow = static_cast<size_t>(q0 + r / a.G) * a.H + kv * a.G + r % a.G;
    if (a.num_splits == 1) {
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
  if (a.num_splits == 1) return;

  // ======================================================== split merge
  // Publish this split and count arrivals; the last CTA of the unit merges all
  // splits (log2-sum-exp weights) and resets the counter for the next call.
  __threadfence();
  consumer_sync();
  uint32_t* counter =
      a.counters + (static_cast<size_t>(b) * a.Hk + kv) * a.num_row_groups + rg;
  if (threadIdx.x == 0) {
    const uint32_t prev = atomicAdd(counter, 1u);
    *sm_flag = (prev == static_cast<uint32_t>(a.num_splits - 1)) ? 1 : 0;
  }
  consumer_sync();
  if (*sm_flag == 0) return;
  __threadfence();
  const size_t stride = static_cast<size_t>(a.total_q) * a.H;
  const int S = a.num_splits;
  float* wts = epi;  // [S][kRows] merge weights, reusing the stage memory
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
    const int d = (idx % (D / 2)) * 2;
    const int r = row0 + row;
    const size_t orow = static_cast<size_t>(q0 + r / a.G) * a.H + kv * a.G + r % a.G;
    const float* base = a.o_part + orow * D + d;
    float s0 = 0.f, s1 = 0.f;
    for (int s8 = 0; s8 < S; s8 += 8) {
      float2 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = (s8 + u < S) ? __ldcg(reinterpret_cast<const float2*>(base + (s8 + u) * stride * D))
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
      *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(a.out) + orow * D + d) =
          __floats2bfloat162_rn(s0, s1);
    else
      *reinterpret_cast<__half2*>(reinterpret_cast<__half*>(a.out) + orow * D + d) =
          __floats2half2_rn(s0, s1);
  }
  if (threadIdx.x == 0) *counter = 0u;  // ready for the next call
}

template <int KV, int D, int BS, int NT, bool LOPACK>
static cudaError_t launch_t(const CUtensorMap& kmap, const CUtensorMap& vmap, const FwdArgs& a,
                            cudaStream_t stream) {
  using C = Cfg<KV, D, BS, NT, LOPACK>;
  auto kern = pa_fwd_kernel<KV, D, BS, NT, LOPACK>;
  // The dynamic shared-memory opt-in is a per-device function attribute: set it
  // the first time this instantiation launches on a device.
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit == 0 || !(configured.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  dim3 grid(a.Hk * a.num_row_groups, a.batch, a.num_splits);
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
