// pa_attention.cu -- fused paged quantised-KV GQA attention for sm_100a.
//
// One CTA owns one (KV head, group of query rows, sequence, KV split).  Its rows
// are (new token, query head of the group) pairs of one sequence, so every row
// reads the same keys: the GQA group x new tokens form the dense N side of the
// tensor-core tile, keys form the M side ("swap-AB"), channels the K side.
//
// Data path per KV block (block_size keys of one head):
//   producer warp : block_table -> two 3-D TMA boxes (K rows, V rows) into a
//                   swizzled shared-memory stage, completion on an mbarrier
//   consumer warp : ldmatrix (K) -> exact code->fp16 conversion in registers ->
//                   mma.sync m16n8k16 against the scale-folded fp16 queries
//                   (fp32 accumulators) -> online softmax in the exp2 domain
//                   (warp shuffles) -> P^T to fp16 with movmatrix ->
//                   ldmatrix.trans (V) -> conversion -> mma.sync into O^T.
// The four consumer warps take alternate blocks and merge (m, l, O) through
// shared memory at the end; the per-channel V scale is applied once there.
// With num_splits > 1 the merged, normalised partial and its log2-sum-exp go
// to the workspace and pa_combine_kernel merges the splits.
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

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

template <int KV, int D, int BS, int NT>
struct Cfg {
  static constexpr int kCHS = (KV == PA_KV_INT4) ? D / 2 : D;  // cache bytes per row
  static constexpr int kTile = BS * kCHS;                       // one block, one head
  static constexpr int kStageBytes = 2 * kTile;                 // K + V
  static constexpr int kChunks = kCHS / 16;                     // 16-byte chunks per row
  static constexpr int kSwzMask = (kCHS == 128) ? 7 : (kCHS == 64) ? 3 : 1;
  static constexpr int kKSteps = D / 16;                        // QK k-steps
  static constexpr int kMTiles = D / 16;                        // PV m-tiles (output dims)
  static constexpr int kKeyTiles = BS / 16;
  static constexpr int kWarps = 4;                              // consumer warps
  static constexpr int kThreads = (kWarps + 1) * 32;            // + one producer warp
  static constexpr int kStagesRaw = 32768 / kStageBytes;
  static constexpr int kStages = kStagesRaw < 8 ? 8 : ((kStagesRaw + 3) / 4) * 4;
  static constexpr int kRows = 8 * NT;
  static constexpr int kPipeBytes = kStages * kStageBytes;
  static constexpr int kEpiBytes = kWarps * kRows * D * 4;
  static constexpr int kDataBytes = kPipeBytes > kEpiBytes ? kPipeBytes : kEpiBytes;
  static constexpr int kBarBytes = 2 * kStages * 8;
  static constexpr int kStatBytes = 2 * kWarps * kRows * 4;
  static constexpr int kSmemBytes = 1024 + kDataBytes + kBarBytes + kStatBytes;
  static_assert(kChunks % 2 == 0, "ldmatrix.x4 covers two 16-byte chunks");
  static_assert(kStages % kWarps == 0, "each stage belongs to one consumer warp");
  static_assert(kTile % ((kSwzMask + 1) * 128) == 0, "tiles keep the swizzle-atom alignment");
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

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

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

template <int KV, int D, int BS, int NT>
__global__ void __launch_bounds__(Cfg<KV, D, BS, NT>::kThreads)
    pa_fwd_kernel(const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap, const FwdArgs a) {
  using C = Cfg<KV, D, BS, NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kDataBytes);  // full | empty
  float* sm_m = reinterpret_cast<float*>(smem + C::kDataBytes + C::kBarBytes);
  float* sm_l = sm_m + C::kWarps * C::kRows;
  float* epi = reinterpret_cast<float*>(smem);  // aliases the stages after the loop

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
  const int row0 = rg * C::kRows;
  if (row0 >= R) return;  // zero new tokens, or fewer rows than this row group
  const int past = Lb - qb;
  const int i_first = row0 / a.G;
  const int i_last = min(R - 1, row0 + C::kRows - 1) / a.G;
  const int kmax = a.causal ? past + i_last + 1 : Lb;       // keys seen by some row
  const int kfull = a.causal ? past + i_first + 1 : Lb;     // keys seen by every row
  const int nblk = (kmax + BS - 1) / BS;
  const int blk_begin = split * a.blocks_per_split;
  const int blk_end = min(nblk, blk_begin + a.blocks_per_split);
  const int nloc = max(0, blk_end - blk_begin);

  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + C::kStages + s); };
  auto k_tile = [&](int s) { return smem + s * C::kStageBytes; };
  auto v_tile = [&](int s) { return smem + s * C::kStageBytes + C::kTile; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_fence_init();
  }
  __syncthreads();

  // ======================================================== producer warp
  if (warp == C::kWarps) {
    if (nloc == 0) return;
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
    }
    const uint64_t policy = l2_evict_first_policy();
    const int32_t* bt = a.block_table + static_cast<size_t>(b) * a.maxb + blk_begin;
    int issued = 0;
    bool ok = true;
    for (int base = 0; base < nloc && ok; base += 32) {
      int phys = 0;
      if (base + lane < nloc) {
        phys = __ldg(bt + base + lane);
        if (phys < 0 || phys >= a.num_blocks) {
          record_error(a.err, PA_DEVERR_BAD_BLOCK);
          phys = a.num_blocks;  // out-of-range box: TMA fills zeros, nothing faults
        }
      }
      const int cnt = min(32, nloc - base);
      for (int j = 0; j < cnt; ++j) {
        const int p = __shfl_sync(0xffffffffu, phys, j);
        if (lane == 0) {
          const int lb = base + j;
          const int s = lb % C::kStages;
          const int round = lb / C::kStages;
          if (round > 0 && !mbar_wait(empty_bar(s), (round - 1) & 1)) {
            record_error(a.err, PA_DEVERR_TIMEOUT);
            ok = false;
          } else {
            mbar_arrive_expect_tx(full_bar(s), C::kStageBytes);
            tma_load_3d(smem_u32(k_tile(s)), &kmap, full_bar(s), 0, kv, p * BS, policy);
            tma_load_3d(smem_u32(v_tile(s)), &vmap, full_bar(s), 0, kv, p * BS, policy);
            ++issued;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
    }
    // Leave no copy in flight: wait for the last box of every stage, all of
    // them within one bounded window.
    if (lane == 0) {
      const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
      for (int s = 0; s < C::kStages && s < issued; ++s) {
        const int last_round = (issued - 1 - s) / C::kStages;
        if (!mbar_wait_until(full_bar(s), last_round & 1, deadline)) {
          record_error(a.err, PA_DEVERR_TIMEOUT);
          break;
        }
      }
    }
    return;
  }

  // ======================================================== consumer warps
  // ---- prologue: fold the K scale into the queries.  q'[d] = q[d] * k_scale[d]
  // / 2^e_kv (2^e_kv: power of two of max |k_scale| of this head), then a second
  // power of two per row keeps |q'| < 1 for any finite input before rounding to
  // fp16; both powers move into the per-row logit multiplier c (exp2 domain).
  float ksmax = 0.f;
  for (int d = lane; d < D; d += 32) ksmax = fmaxf(ksmax, fabsf(a.k_scale[kv * D + d]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ksmax = fmaxf(ksmax, __shfl_xor_sync(0xffffffffu, ksmax, o));
  if (!isfinite(ksmax)) {
    if (warp == 0 && lane == 0) record_error(a.err, PA_DEVERR_BAD_SCALE);
  }
  int e_kv = 0;
  (void)frexpf(ksmax, &e_kv);

  uint32_t qf[NT][C::kKSteps][2];
  float crow[NT][2];
  int lim[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int r = row0 + nt * 8 + g;  // query row of B-operand column g
    const bool valid = r < R;
    const int tok = q0 + (valid ? r / a.G : 0);
    const int head = kv * a.G + (valid ? r % a.G : 0);
    const size_t qoff = (static_cast<size_t>(tok) * a.H + head) * D;
    float w[C::kKSteps][4];
    float rmax = 0.f;
#pragma unroll
    for (int s = 0; s < C::kKSteps; ++s) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int ch = q_channel<KV>(s, j, tig);
        float x = 0.f;
        if (valid) {
          x = a.q_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.q)[qoff + ch])
                       : __half2float(reinterpret_cast<const __half*>(a.q)[qoff + ch]);
        }
        w[s][j] = x * ldexpf(a.k_scale[kv * D + ch], -e_kv);
        rmax = fmaxf(rmax, fabsf(w[s][j]));
      }
    }
    rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 1));
    rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 2));
    int e_q = 0;
    (void)frexpf(rmax, &e_q);
#pragma unroll
    for (int s = 0; s < C::kKSteps; ++s) {
      qf[nt][s][0] = pack_f32x2_to_h2(ldexpf(w[s][0], -e_q), ldexpf(w[s][1], -e_q));
      qf[nt][s][1] = pack_f32x2_to_h2(ldexpf(w[s][2], -e_q), ldexpf(w[s][3], -e_q));
    }
    const float c_mine = ldexpf(a.sm_scale_log2, e_kv + e_q);
    crow[nt][0] = __shfl_sync(0xffffffffu, c_mine, (2 * tig) * 4);
    crow[nt][1] = __shfl_sync(0xffffffffu, c_mine, (2 * tig + 1) * 4);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int rr = row0 + nt * 8 + 2 * tig + j;
      lim[nt][j] = (rr < R && a.causal) ? past + rr / a.G : kmax - 1;
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
  // of the 16-row key tile and chunk (2 cp + (m >> 1)).
  const int lm = lane >> 3;
  const int ld_row = (lane & 7) + 8 * (lm & 1);
  const int ld_chunk = lm >> 1;

  for (int lb = warp; lb < nloc; lb += C::kWarps) {
    const int s = lb % C::kStages;
    if (!mbar_wait(full_bar(s), (lb / C::kStages) & 1)) {
      if (lane == 0) record_error(a.err, PA_DEVERR_TIMEOUT);
      break;
    }
    const uint32_t kbase = smem_u32(k_tile(s));
    const uint32_t vbase = smem_u32(v_tile(s));
    const int key0 = (blk_begin + lb) * BS;
    const bool need_mask = key0 + BS > kfull;
    const bool tail = key0 + BS > Lb;

#pragma unroll
    for (int kt = 0; kt < C::kKeyTiles; ++kt) {
      // ---------------- S^T[key, row] = K q'^T
      float sacc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
      for (int cp = 0; cp < C::kChunks / 2; ++cp) {
        uint32_t r[4];
        const uint32_t off = (kt * 16 + ld_row) * C::kCHS + (2 * cp + ld_chunk) * 16;
        ldsm_x4(kbase + swz<C::kSwzMask>(off), r);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t x0 = r[2 * h], x1 = r[2 * h + 1];  // rows g, g+8 of chunk 2cp+h
          const int c = 2 * cp + h;
          if constexpr (KV == PA_KV_INT8) {
            const uint32_t y0 = x0 ^ 0x80808080u, y1 = x1 ^ 0x80808080u;
            const uint32_t a0 = i8x2_to_h2(y0, 0x4140), a1 = i8x2_to_h2(y1, 0x4140);
            const uint32_t a2 = i8x2_to_h2(y0, 0x4342), a3 = i8x2_to_h2(y1, 0x4342);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              mma_16816(sacc[nt], a0, a1, a2, a3, qf[nt][c][0], qf[nt][c][1]);
          } else if constexpr (KV == PA_KV_FP8_E4M3) {
            const uint32_t a0 = e4m3x2_to_h2(x0), a1 = e4m3x2_to_h2(x1);
            const uint32_t a2 = e4m3x2_to_h2(x0 >> 16), a3 = e4m3x2_to_h2(x1 >> 16);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              mma_16816(sacc[nt], a0, a1, a2, a3, qf[nt][c][0], qf[nt][c][1]);
          } else {  // INT4: one 16-byte chunk = 32 channels = two k-steps
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint32_t z0 = x0 >> (8 * hh), z1 = x1 >> (8 * hh);
              const uint32_t a0 = i4lo_to_h2(z0), a1 = i4lo_to_h2(z1);
              const uint32_t a2 = i4hi_to_h2(z0), a3 = i4hi_to_h2(z1);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                mma_16816(sacc[nt], a0, a1, a2, a3, qf[nt][2 * c + hh][0],
                          qf[nt][2 * c + hh][1]);
            }
          }
        }
      }

      // ---------------- online softmax (exp2 domain)
      float pv[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = e & 1;
          float x = sacc[nt][e] * crow[nt][j];
          if (need_mask) {
            const int key = key0 + kt * 16 + g + (e >> 1) * 8;
            if (key > lim[nt][j]) x = -INFINITY;
          }
          pv[nt][e] = x;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float mx = fmaxf(pv[nt][j], pv[nt][j + 2]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float m_new = fmaxf(m_run[nt][j], mx);
          const float m_ref = (m_new == -INFINITY) ? 0.f : m_new;
          const float alpha = fast_exp2(m_run[nt][j] - m_ref);
          m_run[nt][j] = m_new;
          const float p0 = fast_exp2(pv[nt][j] - m_ref);
          const float p1 = fast_exp2(pv[nt][j + 2] - m_ref);
          pv[nt][j] = p0;
          pv[nt][j + 2] = p1;
          l_run[nt][j] = l_run[nt][j] * alpha + (p0 + p1);
#pragma unroll
          for (int mt = 0; mt < C::kMTiles; ++mt) {
            o[nt][mt][j] *= alpha;
            o[nt][mt][j + 2] *= alpha;
          }
        }
      }

      // ---------------- P^T as the B operand: (key g; rows 2tig, 2tig+1) -> (keys; row g)
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        pb[nt][0] = movmatrix_trans(pack_f32x2_to_h2(pv[nt][0], pv[nt][1]));
        pb[nt][1] = movmatrix_trans(pack_f32x2_to_h2(pv[nt][2], pv[nt][3]));
      }

      // Keys past the sequence end in the last block hold stale bytes; an FP8 NaN
      // there would poison P*V even with P = 0, so such V codes are zeroed.
      uint32_t vmask_lo = 0xffffffffu, vmask_hi = 0xffffffffu;
      if constexpr (KV == PA_KV_FP8_E4M3) {
        if (tail) {
          const int kb = key0 + kt * 16 + 2 * tig;
          vmask_lo = (kb < Lb ? 0x0000ffffu : 0u) | (kb + 1 < Lb ? 0xffff0000u : 0u);
          vmask_hi = (kb + 8 < Lb ? 0x0000ffffu : 0u) | (kb + 9 < Lb ? 0xffff0000u : 0u);
        }
      }

      // ---------------- O^T[dim, row] += V^T P^T
#pragma unroll
      for (int cp = 0; cp < C::kChunks / 2; ++cp) {
        uint32_t r[4];
        const uint32_t off = (kt * 16 + ld_row) * C::kCHS + (2 * cp + ld_chunk) * 16;
        ldsm_x4_trans(vbase + swz<C::kSwzMask>(off), r);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t lo = r[2 * h], hi = r[2 * h + 1];  // keys 2tig.. / 2tig+8.. of chunk c
          const int c = 2 * cp + h;
          if constexpr (KV == PA_KV_INT8) {
            const uint32_t ylo = lo ^ 0x80808080u, yhi = hi ^ 0x80808080u;
            const uint32_t a0 = i8x2_to_h2(ylo, 0x4240), a1 = i8x2_to_h2(ylo, 0x4341);
            const uint32_t a2 = i8x2_to_h2(yhi, 0x4240), a3 = i8x2_to_h2(yhi, 0x4341);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_16816(o[nt][c], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
          } else if constexpr (KV == PA_KV_FP8_E4M3) {
            const uint32_t zlo = prmt(lo, 0u, 0x3120), zhi = prmt(hi, 0u, 0x3120);
            const uint32_t a0 = e4m3x2_to_h2(zlo) & vmask_lo, a1 = e4m3x2_to_h2(zlo >> 16) & vmask_lo;
            const uint32_t a2 = e4m3x2_to_h2(zhi) & vmask_hi, a3 = e4m3x2_to_h2(zhi >> 16) & vmask_hi;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_16816(o[nt][c], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
          } else {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint32_t zl = lo >> (8 * hh), zh = hi >> (8 * hh);
              const uint32_t a0 = i4lo_to_h2(zl), a1 = i4hi_to_h2(zl);
              const uint32_t a2 = i4lo_to_h2(zh), a3 = i4hi_to_h2(zh);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                mma_16816(o[nt][2 * c + hh], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));
  }

  // ======================================================== merge the warps
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float l = l_run[nt][j];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      l_run[nt][j] = l;
      if (g == 0) {
        sm_m[warp * C::kRows + nt * 8 + 2 * tig + j] = m_run[nt][j];
        sm_l[warp * C::kRows + nt * 8 + 2 * tig + j] = l;
      }
    }
  consumer_sync();  // all warps left the pipeline: the stages may be reused
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int row = nt * 8 + 2 * tig + j;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < C::kWarps; ++w) M = fmaxf(M, sm_m[w * C::kRows + row]);
      const float f = (m_run[nt][j] == -INFINITY) ? 0.f : fast_exp2(m_run[nt][j] - M);
#pragma unroll
      for (int mt = 0; mt < C::kMTiles; ++mt) {
        const int d = out_dim<KV>(mt, g);
        float2 v;
        v.x = o[nt][mt][j] * f;
        v.y = o[nt][mt][j + 2] * f;
        *reinterpret_cast<float2*>(epi + (warp * C::kRows + row) * D + d) = v;
      }
    }
  consumer_sync();

  const int nthr = C::kWarps * 32;
  for (int idx = threadIdx.x; idx < C::kRows * (D / 2); idx += nthr) {
    const int row = idx / (D / 2);
    const int d = (idx % (D / 2)) * 2;
    const int r = row0 + row;
    if (r >= R) continue;
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
    const float o0 = s0 * inv * a.v_scale[kv * D + d];
    const float o1 = s1 * inv * a.v_scale[kv * D + d + 1];
    const int tok = q0 + r / a.G;
    const int head = kv * a.G + r % a.G;
    const size_t orow = static_cast<size_t>(tok) * a.H + head;
    if (a.num_splits == 1) {
      if (a.out_bf16) {
        *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(a.out) + orow * D + d) =
            __floats2bfloat162_rn(o0, o1);
      } else {
        *reinterpret_cast<__half2*>(reinterpret_cast<__half*>(a.out) + orow * D + d) =
            __floats2half2_rn(o0, o1);
      }
    } else {
      const size_t prow = static_cast<size_t>(split) * a.total_q * a.H + orow;
      *reinterpret_cast<float2*>(a.o_part + prow * D + d) = make_float2(o0, o1);
      if (d == 0) a.lse_part[prow] = (L > 0.f) ? M + __log2f(L) : -INFINITY;
    }
  }
}

// Log-sum-exp merge of the KV splits (exp2 domain):
// out = sum_s 2^(lse_s - M) o_s / sum_s 2^(lse_s - M), M = max_s lse_s.
__global__ void __launch_bounds__(128) pa_combine_kernel(const CombineArgs a) {
  const int kv = blockIdx.x, b = blockIdx.y;
  const int q0 = a.cu_seqlens_q[b];
  const int qb = a.cu_seqlens_q[b + 1] - q0;
  if (q0 < 0 || qb < 0 || q0 + qb > a.total_q) return;  // the forward kernel flagged it
  const int R = qb * a.G;
  const int D = a.D;
  const size_t stride = static_cast<size_t>(a.total_q) * a.H;
  for (int idx = threadIdx.x; idx < R * (D / 2); idx += blockDim.x) {
    const int r = idx / (D / 2);
    const int d = (idx % (D / 2)) * 2;
    const size_t orow = static_cast<size_t>(q0 + r / a.G) * a.H + kv * a.G + r % a.G;
    float M = -INFINITY;
    for (int s = 0; s < a.num_splits; ++s) M = fmaxf(M, a.lse_part[s * stride + orow]);
    float wsum = 0.f, s0 = 0.f, s1 = 0.f;
    if (M != -INFINITY) {
      for (int s = 0; s < a.num_splits; ++s) {
        const float ls = a.lse_part[s * stride + orow];
        if (ls == -INFINITY) continue;
        const float w = fast_exp2(ls - M);
        const float2 v = *reinterpret_cast<const float2*>(a.o_part + (s * stride + orow) * D + d);
        wsum += w;
        s0 += w * v.x;
        s1 += w * v.y;
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    if (a.out_bf16) {
      *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(a.out) + orow * D + d) =
          __floats2bfloat162_rn(s0 * inv, s1 * inv);
    } else {
      *reinterpret_cast<__half2*>(reinterpret_cast<__half*>(a.out) + orow * D + d) =
          __floats2half2_rn(s0 * inv, s1 * inv);
    }
  }
}

template <int KV, int D, int BS, int NT>
static cudaError_t launch_t(const CUtensorMap& kmap, const CUtensorMap& vmap, const FwdArgs& a,
                            cudaStream_t stream) {
  using C = Cfg<KV, D, BS, NT>;
  auto kern = pa_fwd_kernel<KV, D, BS, NT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(a.Hk * a.num_row_groups, a.batch, a.num_splits);
  kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(kmap, vmap, a);
  return cudaGetLastError();
}

template <int KV, int D, int BS, int NT>
static int smem_t() {
  return Cfg<KV, D, BS, NT>::kSmemBytes;
}

#define PA_DISPATCH(FN, ...)                                                          \
  do {                                                                                \
    const int nt = rows_per_cta == 16 ? 2 : 1;                                        \
    switch (kv_dtype * 1000 + head_size * 10 + (block_size == 32 ? 1 : 0) * 100 + nt) { \
      case PA_KV_INT8 * 1000 + 640 + 1: return FN<PA_KV_INT8, 64, 16, 1>(__VA_ARGS__);    \
      case PA_KV_INT8 * 1000 + 640 + 2: return FN<PA_KV_INT8, 64, 16, 2>(__VA_ARGS__);    \
      case PA_KV_INT8 * 1000 + 740 + 1: return FN<PA_KV_INT8, 64, 32, 1>(__VA_ARGS__);    \
      case PA_KV_INT8 * 1000 + 740 + 2: return FN<PA_KV_INT8, 64, 32, 2>(__VA_ARGS__);    \
      case PA_KV_INT8 * 1000 + 1280 + 1: return FN<PA_KV_INT8, 128, 16, 1>(__VA_ARGS__);  \
      case PA_KV_INT8 * 1000 + 1280 + 2: return FN<PA_KV_INT8, 128, 16, 2>(__VA_ARGS__);  \
      case PA_KV_INT8 * 1000 + 1380 + 1: return FN<PA_KV_INT8, 128, 32, 1>(__VA_ARGS__);  \
      case PA_KV_INT8 * 1000 + 1380 + 2: return FN<PA_KV_INT8, 128, 32, 2>(__VA_ARGS__);  \
      case PA_KV_INT4 * 1000 + 640 + 1: return FN<PA_KV_INT4, 64, 16, 1>(__VA_ARGS__);    \
      case PA_KV_INT4 * 1000 + 640 + 2: return FN<PA_KV_INT4, 64, 16, 2>(__VA_ARGS__);    \
      case PA_KV_INT4 * 1000 + 740 + 1: return FN<PA_KV_INT4, 64, 32, 1>(__VA_ARGS__);    \
      case PA_KV_INT4 * 1000 + 740 + 2: return FN<PA_KV_INT4, 64, 32, 2>(__VA_ARGS__);    \
      case PA_KV_INT4 * 1000 + 1280 + 1: return FN<PA_KV_INT4, 128, 16, 1>(__VA_ARGS__);  \
      case PA_KV_INT4 * 1000 + 1280 + 2: return FN<PA_KV_INT4, 128, 16, 2>(__VA_ARGS__);  \
      case PA_KV_INT4 * 1000 + 1380 + 1: return FN<PA_KV_INT4, 128, 32, 1>(__VA_ARGS__);  \
      case PA_KV_INT4 * 1000 + 1380 + 2: return FN<PA_KV_INT4, 128, 32, 2>(__VA_ARGS__);  \
      case PA_KV_FP8_E4M3 * 1000 + 640 + 1: return FN<PA_KV_FP8_E4M3, 64, 16, 1>(__VA_ARGS__);   \
      case PA_KV_FP8_E4M3 * 1000 + 640 + 2: return FN<PA_KV_FP8_E4M3, 64, 16, 2>(__VA_ARGS__);   \
      case PA_KV_FP8_E4M3 * 1000 + 740 + 1: return FN<PA_KV_FP8_E4M3, 64, 32, 1>(__VA_ARGS__);   \
      case PA_KV_FP8_E4M3 * 1000 + 740 + 2: return FN<PA_KV_FP8_E4M3, 64, 32, 2>(__VA_ARGS__);   \
      case PA_KV_FP8_E4M3 * 1000 + 1280 + 1: return FN<PA_KV_FP8_E4M3, 128, 16, 1>(__VA_ARGS__); \
      case PA_KV_FP8_E4M3 * 1000 + 1280 + 2: return FN<PA_KV_FP8_E4M3, 128, 16, 2>(__VA_ARGS__); \
      case PA_KV_FP8_E4M3 * 1000 + 1380 + 1: return FN<PA_KV_FP8_E4M3, 128, 32, 1>(__VA_ARGS__); \
      case PA_KV_FP8_E4M3 * 1000 + 1380 + 2: return FN<PA_KV_FP8_E4M3, 128, 32, 2>(__VA_ARGS__); \
      default: break;                                                                 \
    }                                                                                 \
  } while (0)

cudaError_t launch_forward(int kv_dtype, int head_size, int block_size, int rows_per_cta,
                           const CUtensorMap& kmap, const CUtensorMap& vmap, const FwdArgs& a,
                           cudaStream_t stream) {
  PA_DISPATCH(launch_t, kmap, vmap, a, stream);
  return cudaErrorInvalidValue;
}

int forward_smem_bytes(int kv_dtype, int head_size, int block_size, int rows_per_cta) {
  PA_DISPATCH(smem_t);
  return -1;
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
  dim3 grid(a.Hk, a.batch);
  pa_combine_kernel<<<grid, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace pa
