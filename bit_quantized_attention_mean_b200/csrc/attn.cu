// attn.cu -- fused 8-bit attention forward for sm_100a (B200).
//
// Follows the SageAttention article (method section: the per-block INT8
// quantization step and the FP16 P V step): S = Q_i8 K_i8^T with an INT32
// accumulator, dequantized by q_scale * k_scale, softmax over
// FlashAttention-style tiles, and O = P V with P and V in FP16.
// sm_scale * log2(e) is already in q_scale, so the softmax runs in base 2
// (exp2).
//
// One CTA owns one 128-row Q tile (the Q quantization block) and walks the
// 64-row K/V tiles (the K quantization block) of its (batch, kv head):
//
//   warp 4      TMA producer: Q tile once, then K (int8) and V (fp16) tiles
//               into a 3-stage shared-memory ring (no multicast).
//   warp 5      MMA issuer (one thread): S_j = Q K_j^T with tcgen05.mma
//               kind::i8 into tensor memory (int32, double-buffered), then
//               O += P_j V_j with kind::f16, A = P read from tensor memory,
//               B = V from shared memory (MN-major), O in fp32 tensor memory.
//   warps 0-3   softmax: thread t owns row t.  tcgen05.ld of its 64 scores,
//               integer row max, exact int->float, one FFMA per score for the
//               dequantization and max shift, ex2, fp16 pack, tcgen05.st of P
//               over the consumed scores.  O is rescaled in tensor memory only
//               when the running max grows by more than 2^8 (the result does
//               not depend on the reference point, only the fp16 range does).
//
// The MMA thread issues S_{j+1} before P_j V_j so the tensor core computes the
// next scores while the softmax warps work; two CTAs share each SM (256 of the
// 512 tensor-memory columns each), so one CTA's softmax overlaps the other's
// MMAs.  tcgen05 operations from one thread execute in issue order, which is
// what makes reusing a score buffer for S_{j+2} after P_j V_j safe.
//
// F16ACC selects the accumulator the article names for P V (an fp16
// accumulator, method section, FP16 P V step): the P V products accumulate in fp16 (one value
// per tensor-memory column, in its low half), and the running max is exact
// (O rescaled whenever it grows) so that P <= 1 keeps the sums in fp16 range.
// The default accumulates in fp32.
//
// At d = 64 (fp16 P V, fp32 sums) P V runs with N = d + 16 against V and a
// constant tile whose first column is all ones, so the accumulator's column d
// is each row's sum of the same fp16 P the MMA used, and the softmax warps
// keep no row sum of their own.
//
// Tensor memory (256 columns): [0,64) S/P buffer 0, [64,128) S/P buffer 1,
// [128,128+d) O accumulator (+16 columns, the row sums, at d = 64).  Every
// mbarrier wait is bounded (2 s); on expiry the CTA stops issuing work, drains
// what is in flight, frees its tensor memory and records the failing site in
// the device status word.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cstdint>
#include <mutex>

#include "sage_internal.h"
#include "sm100_ptx.cuh"

namespace sage {

__device__ int g_device_status;

constexpr long long kGlobalOrderKVBytes = 112ll << 20;  // K/V total that stays L2-resident
constexpr int BQ = 128;  // query rows per tile  (= Q quantization block)
constexpr int BK = 64;   // key rows per tile    (= K quantization block)

// P V variants: fp16 P and V with fp32 sums (default), fp16 sums, or P and V
// in E4M3 with fp32 sums.
enum PvMode : int { kPvF32 = 0, kPvF16Acc = 1, kPvFp8 = 2 };

template <int D, bool FP8V = false, bool ONES = false>
struct AttnCfg {
  static constexpr int STAGES = 3;
  static constexpr int Q_BYTES = BQ * D;      // int8
  static constexpr int K_BYTES = BK * D;      // int8, per stage
  // per stage: fp16 V [64 keys x D], or E4M3 V^T [D channels x 64 keys]
  static constexpr int V_BYTES = FP8V ? BK * D : BK * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * K_BYTES;
  // ONES: a constant [64 keys x 64] fp16 tile whose first column is 1, read
  // as 16 more B columns of P V, so the tensor core also sums P per row
  static constexpr int OFF_ONES = OFF_V + STAGES * V_BYTES;
  static constexpr int OFF_BAR = OFF_ONES + (ONES ? BK * 128 : 0);
  // barrier slots
  static constexpr int B_Q_FULL = 0;
  static constexpr int B_K_FULL = 1;
  static constexpr int B_V_FULL = B_K_FULL + STAGES;
  static constexpr int B_KV_EMPTY = B_V_FULL + STAGES;
  static constexpr int B_S_FULL = B_KV_EMPTY + STAGES;
  static constexpr int B_P_FULL = B_S_FULL + 2;
  static constexpr int B_O_DONE = B_P_FULL + 2;
  static constexpr int B_O_FINAL = B_O_DONE + 1;
  static constexpr int B_TEARDOWN = B_O_FINAL + 1;
  static constexpr int NUM_BARS = B_TEARDOWN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int USED = OFF_MISC + 16;
  // pad so at most two CTAs fit per SM (tensor memory holds two allocations)
  static constexpr int SMEM_BYTES = (USED + 1024) > 80 * 1024 ? (USED + 1024) : 80 * 1024;
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t S_COL = 0;  // buffer b at S_COL + 64 * b
  static constexpr uint32_t O_COL = 128;
  // Q/K int8 rows are D bytes: 128B swizzle for d=128, 64B for d=64; the
  // 8-row core-matrix groups are 8*D bytes apart.
  static constexpr uint32_t QK_SWIZZLE = D == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t QK_SBO = 8 * D;
  static_assert(Q_BYTES % 1024 == 0 && K_BYTES % 1024 == 0 && V_BYTES % 1024 == 0,
                "tiles must stay 1024-byte aligned");
};

// An accumulator column as fp32: fp32 sums hold the value itself, fp16 sums
// an fp16 value in the low half.
template <bool F16ACC>
__device__ __forceinline__ float acc_value(uint32_t col) {
  return F16ACC ? __half2float(__ushort_as_half((unsigned short)(col & 0xffffu))) : __uint_as_float(col);
}

// An fp16 accumulator column multiplied by alpha (rounded back to fp16).
__device__ __forceinline__ uint32_t acc16_scale(uint32_t col, float alpha) {
  return (uint32_t)__half_as_ushort(__float2half_rn(acc_value<true>(col) * alpha));
}

// Warp-uniform bounded wait: every lane waits, then the warp agrees.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int site, uint64_t limit_ns = kWaitLimitNs) {
  const bool ok = mbar_wait(bar, parity, abort_flag, &g_device_status, site, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

template <int D, bool CAUSAL, int PV>
__global__ void __launch_bounds__(192, 2)
sage_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ q_scale,
                     const float* __restrict__ k_scale, const float* __restrict__ v_scale,
                     __half* __restrict__ out, int H, int Hkv, int Lq, int Lk, int nqt,
                     int global_lpt, int qbr, const int* __restrict__ seqlens_q,
                     const int* __restrict__ seqlens_k) {
  constexpr bool F16ACC = PV == kPvF16Acc;
  constexpr bool FP8V = PV == kPvFp8;
  // d = 64, fp16 P V with fp32 sums: the row sums of P come from the tensor
  // core (16 extra accumulator columns, the first one the sum)
  constexpr bool ONES = D == 64 && PV == kPvF32;
  constexpr int OW = ONES ? D + 16 : D;  // accumulator columns of P V
  using C = AttnCfg<D, FP8V, ONES>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment of the shared-window address (swizzle atoms)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Causal tiles differ in length; launch the longest first.  When the K/V
  // of every head fit in L2 together, order across heads (global longest
  // first); otherwise keep each head's tiles together so its K/V stay hot.
  int bh, qt;
  if (CAUSAL && global_lpt) {
    const int BH = gridDim.x / nqt;
    qt = nqt - 1 - (int)(blockIdx.x / BH);
    bh = blockIdx.x - (nqt - 1 - qt) * BH;
  } else {
    bh = blockIdx.x / nqt;
    qt = blockIdx.x - bh * nqt;
    if (CAUSAL) qt = nqt - 1 - qt;  // longest rows first within a head
  }
  const int h = bh % H, b = bh / H;
  const int bhk = b * Hkv + h / (H / Hkv);
  const int q0 = qt * BQ;
  const int nkb = (Lk + BK - 1) / BK;  // k_scale row length
  // rows and keys of this batch entry: all of them, or its own counts in a
  // padded batch (rows past Lqb are written as zeros)
  const int Lqb = seqlens_q ? min(max(__ldg(seqlens_q + b), 0), Lq) : Lq;
  const int Lkb = seqlens_k ? min(max(__ldg(seqlens_k + b), 0), Lk) : Lk;
  int nkt = q0 < Lqb ? (Lkb + BK - 1) / BK : 0;
  if (CAUSAL && nkt > 0) {
    const int last_row = min(q0 + BQ, Lqb) - 1;
    const int vis = last_row + (Lkb - Lqb) + 1;  // keys [0, vis) visible to the tile's last row
    nkt = vis <= 0 ? 0 : min(nkt, (vis + BK - 1) / BK);
  }

  if (tid == 0) {
    for (int i = 0; i < C::NUM_BARS; ++i)
      mbar_init(&bars[i], (i == C::B_P_FULL || i == C::B_P_FULL + 1) ? 128u : 1u);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if constexpr (ONES) {
    // key row r holds 128 bytes; its 16-byte chunk c sits at chunk c ^ (r % 8)
    // (128-byte swizzle), so column 0 of row r is at byte r * 128 + (r % 8) * 16
    uint4* ones = reinterpret_cast<uint4*>(smem + C::OFF_ONES);
    for (int i = tid; i < BK * 8; i += blockDim.x) {
      const int r = i >> 3, cchunk = i & 7;
      ones[i] = make_uint4(cchunk == (r & 7) ? 0x3C00u : 0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();  // visible to the tensor core
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nkt > 0) {
      const uint64_t keep = l2_policy_evict_last();    // K/V: re-read by the head's other tiles
      const uint64_t stream = l2_policy_evict_first();  // Q: read once
      mbar_arrive_expect_tx(&bars[C::B_Q_FULL], C::Q_BYTES);
      tma_load_3d_hint(smem + C::OFF_Q, &tm_q, &bars[C::B_Q_FULL], 0, q0, bh, stream);
      int issued = 0;
      for (int j = 0; j < nkt; ++j) {
        const int s = j % C::STAGES;
        if (j >= C::STAGES &&
            !mbar_wait(&bars[C::B_KV_EMPTY + s], ((j / C::STAGES) - 1) & 1, abort_flag,
                       &g_device_status, 1))
          break;
        mbar_arrive_expect_tx(&bars[C::B_K_FULL + s], C::K_BYTES);
        tma_load_3d_hint(smem + C::OFF_K + s * C::K_BYTES, &tm_k, &bars[C::B_K_FULL + s], 0,
                         j * BK, bhk, keep);
        mbar_arrive_expect_tx(&bars[C::B_V_FULL + s], C::V_BYTES);
        if constexpr (FP8V) {
          // E4M3 V^T tile: D channel rows of 64 keys (64-byte swizzle)
          tma_load_3d_hint(smem + C::OFF_V + s * C::V_BYTES, &tm_v, &bars[C::B_V_FULL + s],
                           j * BK, 0, bhk, keep);
        } else {
#pragma unroll
          for (int cc = 0; cc < D / 64; ++cc)
            tma_load_3d_hint(smem + C::OFF_V + s * C::V_BYTES + cc * (BK * 128), &tm_v,
                             &bars[C::B_V_FULL + s], cc * 64, j * BK, bhk, keep);
        }
        issued = j + 1;
      }
      // nothing may still be landing in shared memory when the CTA exits
      mbar_wait_drain(&bars[C::B_Q_FULL], 0);
      for (int j = issued > C::STAGES ? issued - C::STAGES : 0; j < issued; ++j) {
        mbar_wait_drain(&bars[C::B_K_FULL + j % C::STAGES], (j / C::STAGES) & 1);
        mbar_wait_drain(&bars[C::B_V_FULL + j % C::STAGES], (j / C::STAGES) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && nkt > 0) {
      constexpr uint32_t idesc_qk = make_idesc_i8(BQ, BK);
      constexpr uint32_t idesc_pv =
          FP8V ? make_idesc_f8(BQ, D) : make_idesc_f16(BQ, OW, /*b_mn_major=*/true, F16ACC);
      const uint32_t sQ = smem_u32(smem + C::OFF_Q);
      auto issue_pv = [&](int jj) -> bool {
        const int bb = jj & 1, ss = jj % C::STAGES;
        if (!mbar_wait(&bars[C::B_P_FULL + bb], (jj >> 1) & 1, abort_flag, &g_device_status, 2))
          return false;
        if (!mbar_wait(&bars[C::B_V_FULL + ss], (jj / C::STAGES) & 1, abort_flag,
                       &g_device_status, 3))
          return false;
        tc_fence_after_sync();
        const uint32_t sV = smem_u32(smem + C::OFF_V + ss * C::V_BYTES);
        const uint32_t p_tmem = tmem + C::S_COL + 64u * bb;
        if constexpr (FP8V) {
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // V^T tile: K-major B operand, rows of 64 keys (64B swizzle), 8-row
            // groups 512 B apart; 32 keys per MMA; P: 4 keys per column
            const uint64_t bdesc = make_smem_desc(sV + kk * 32, 16, 512, kSwizzle64B);
            umma_f8_ts(tmem + C::O_COL, p_tmem + kk * 8, bdesc, idesc_pv,
                       (jj > 0 || kk > 0) ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // V tile: D/64 chunks of [64 keys x 128 B] (128B swizzle), MN-major
            // B operand; LBO = chunk stride, SBO = 8 key rows; 16 keys per MMA.
            // with ONES the second 64-column atom is the ones tile
            const uint32_t lbo = ONES ? (uint32_t)(C::OFF_ONES - C::OFF_V - ss * C::V_BYTES)
                                      : (uint32_t)(BK * 128);
            const uint64_t bdesc = make_smem_desc(sV + kk * 16 * 128, lbo, 1024, kSwizzle128B);
            umma_f16_ts(tmem + C::O_COL, p_tmem + kk * 8, bdesc, idesc_pv,
                        (jj > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&bars[C::B_KV_EMPTY + ss]);
        umma_commit(&bars[C::B_O_DONE]);
        return true;
      };
      bool ok = mbar_wait(&bars[C::B_Q_FULL], 0, abort_flag, &g_device_status, 4);
      if (ok) {
        tc_fence_after_sync();
        for (int j = 0; j < nkt; ++j) {
          const int s = j % C::STAGES, bb = j & 1;
          if (!mbar_wait(&bars[C::B_K_FULL + s], (j / C::STAGES) & 1, abort_flag,
                         &g_device_status, 5)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sK = smem_u32(smem + C::OFF_K + s * C::K_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            // K-major int8 operands, 32 bytes of K per MMA
            const uint64_t adesc = make_smem_desc(sQ + kk * 32, 16, C::QK_SBO, C::QK_SWIZZLE);
            const uint64_t bdesc = make_smem_desc(sK + kk * 32, 16, C::QK_SBO, C::QK_SWIZZLE);
            umma_i8_ss(tmem + C::S_COL + 64u * bb, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars[C::B_S_FULL + bb]);
          if (j > 0 && !issue_pv(j - 1)) {
            ok = false;
            break;
          }
        }
        if (ok && issue_pv(nkt - 1)) umma_commit(&bars[C::B_O_FINAL]);
      }
      // every issued MMA must be complete before the tensor memory is freed
      umma_commit(&bars[C::B_TEARDOWN]);
      mbar_wait_drain(&bars[C::B_TEARDOWN], 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    const int row = tid;  // warp w reads tensor-memory lanes [32w, 32w+32)
    const int qrow = q0 + row;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    // this row's Q scale (blocks of qbr rows; padding rows reuse the last)
    const int nqs = (Lq + qbr - 1) / qbr;
    const bool real = qrow < Lqb;
    const float sq = real ? __ldg(q_scale + (size_t)bh * nqs + qrow / qbr) : 0.f;
    const float* ks = k_scale + (size_t)bhk * nkb;
    const int diag = real ? qrow + (Lkb - Lqb) + 1 : 0;  // keys [0, diag) visible to this row
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    float ck = nkt > 0 ? __ldg(ks) : 0.f;
    for (int j = 0; j < nkt; ++j) {
      const int bb = j & 1;
      const float c = __fmul_rn(sq, ck);
      if (j + 1 < nkt) ck = __ldg(ks + j + 1);
      if (!warp_wait(&bars[C::B_S_FULL + bb], (j >> 1) & 1, abort_flag, 6)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t s_tmem = tmem + lane_base + C::S_COL + 64u * bb;
      uint32_t s[64];
      tmem_ld64(s_tmem, s);

      int vis = real ? Lkb - j * BK : 0;
      if (CAUSAL) vis = min(vis, diag - j * BK);
      const bool full = vis >= BK;
      int mx = INT_MIN;
      if (full) {
#pragma unroll
        for (int k = 0; k < BK; ++k) mx = max(mx, (int)s[k]);
      } else {
#pragma unroll
        for (int k = 0; k < BK; ++k) mx = (k < vis) ? max(mx, (int)s[k]) : mx;
      }
      // |S| <= 127*127*128 < 2^22, so the int -> float conversion is exact
      const float mt = vis > 0 ? (float)mx * c : -INFINITY;
      // rescale threshold (base 2): lazy for fp32 sums, exact for fp16 sums
      const bool need = mt > m_run + (F16ACC ? 0.0f : 8.0f);
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m_run - mt);  // 0 when m_run = -inf
        m_run = mt;
      }
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // S_j's commit came after P V_{j-2} was issued, so O_DONE is at most
        // one phase behind P V_{j-1}: the parity wait is unambiguous
        if (!warp_wait(&bars[C::B_O_DONE], (j - 1) & 1, abort_flag, 7)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        // (at d = 64 the last 32-column chunk also covers 16 allocated
        // columns past the accumulator, which nothing reads)
#pragma unroll 1
        for (int cc = 0; cc < (OW + 31) / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + C::O_COL + cc * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = F16ACC ? acc16_scale(o[i], alpha)
                                                      : __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem + lane_base + C::O_COL + cc * 32, o);
        }
      }
      l_run *= alpha;
      const float moff = m_run == -INFINITY ? 0.f : m_run;
      uint32_t pk[32];
      float lsum = 0.f;
#pragma unroll
      for (int k = 0; k < BK; k += 2) {
        // |S| <= 127*127*128 < 2^24: the int -> float conversion is exact
        const float x0 = __int2float_rn((int)s[k]);
        const float x1 = __int2float_rn((int)s[k + 1]);
        float p0 = ex2_approx(fmaf(x0, c, -moff));
        float p1 = ex2_approx(fmaf(x1, c, -moff));
        if (!full) {
          p0 = k < vis ? p0 : 0.f;
          p1 = k + 1 < vis ? p1 : 0.f;
        }
        if constexpr (!ONES) lsum += p0 + p1;
        if constexpr (FP8V) {
          // P <= 2^8 (lazy max), so P * 1.75 <= 448 fits E4M3; 4 keys a column
          const uint32_t e = pack_e4m3x2(p0 * 1.75f, p1 * 1.75f);
          pk[k >> 2] = (k & 2) ? (pk[k >> 2] | (e << 16)) : e;
        } else {
          pk[k >> 1] = pack_half2(p0, p1);
        }
      }
      l_run += lsum;
      // P over the consumed scores
      if constexpr (FP8V) tmem_st16(s_tmem, pk);
      else tmem_st32(s_tmem, pk);
      tc_fence_before_sync();
      mbar_arrive(&bars[C::B_P_FULL + bb]);
    }
    if (ok && nkt > 0) {
      // O_DONE may still be two phases behind here (only P V_{nkt-3} is known
      // to be complete), so the final accumulator has its own one-shot barrier
      ok = warp_wait(&bars[C::B_O_FINAL], 0, abort_flag, 8);
      tc_fence_after_sync();
    }
    if (ok) {
      float lsum_all = l_run;
      if constexpr (ONES) {
        // the tensor core's row sum of the fp16 P, column D of the accumulator
        uint32_t o[32];
        if (nkt > 0) tmem_ld32(tmem + lane_base + C::O_COL + D, o);
        lsum_all = nkt > 0 ? __uint_as_float(o[0]) : 0.f;
      }
      const float inv = lsum_all > 0.f ? 1.f / lsum_all : 0.f;
      __half* orow = out + ((size_t)bh * Lq + qrow) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        if (nkt > 0) {
          tmem_ld32(tmem + lane_base + C::O_COL + cc * 32, o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        uint32_t hv[16];
        if constexpr (FP8V) {
          // undo the per-channel V scale and the 1.75 of P
          const float* vs = v_scale + (size_t)bhk * D + cc * 32;
          const float s8 = inv * (1.0f / 1.75f);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            hv[i] = pack_half2(__uint_as_float(o[2 * i]) * (__ldg(vs + 2 * i) * s8),
                               __uint_as_float(o[2 * i + 1]) * (__ldg(vs + 2 * i + 1) * s8));
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            hv[i] = pack_half2(acc_value<F16ACC>(o[2 * i]) * inv,
                               acc_value<F16ACC>(o[2 * i + 1]) * inv);
        }
        if (qrow < Lq) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------- host

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

static bool make_map_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esize,
                        uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box0, uint32_t box1,
                        CUtensorMapSwizzle sw) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * esize, d0 * d1 * esize};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool CAUSAL, int PV>
static cudaError_t launch_attn_t(const AttnArgs& a, cudaStream_t st, int* launches) {
  using C = AttnCfg<D, PV == kPvFp8, D == 64 && PV == kPvF32>;
  auto kern = sage_attn_fwd_kernel<D, CAUSAL, PV>;
  // per device context; cheap enough to repeat on every launch
  cudaError_t attr_err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (attr_err != cudaSuccess) return attr_err;

  CUtensorMap tq, tk, tv;
  const CUtensorMapSwizzle qk_sw =
      D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!make_map_3d(&tq, a.q_i8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, a.Lq, (uint64_t)a.B * a.H, D,
                   BQ, qk_sw) ||
      !make_map_3d(&tk, a.k_i8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, a.Lk, (uint64_t)a.B * a.Hkv,
                   D, BK, qk_sw) ||
      !(PV == kPvFp8
            ? make_map_3d(&tv, a.v8t, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1,
                          (uint64_t)(a.Lk + BK - 1) / BK * BK, D, (uint64_t)a.B * a.Hkv, BK, D,
                          CU_TENSOR_MAP_SWIZZLE_64B)
            : make_map_3d(&tv, a.v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, D, a.Lk,
                          (uint64_t)a.B * a.Hkv, 64, BK, CU_TENSOR_MAP_SWIZZLE_128B)))
    return cudaErrorInvalidValue;

  const int nqt = (a.Lq + BQ - 1) / BQ;
  const long long grid = (long long)a.B * a.H * nqt;
  const long long kv_bytes = (long long)a.B * a.Hkv * a.Lk * D * (PV == kPvFp8 ? 2 : 3);
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  kern<<<(unsigned)grid, 192, C::SMEM_BYTES, st>>>(tq, tk, tv, a.q_scale, a.k_scale, a.v_scale,
                                                   a.out, a.H, a.Hkv, a.Lq, a.Lk, nqt,
                                                   kv_bytes <= kGlobalOrderKVBytes ? 1 : 0,
                                                   a.q_block_rows, a.seqlens_q, a.seqlens_k);
  *launches += 1;
  return cudaGetLastError();
}

template <int PV>
static cudaError_t launch_attn_pv(const AttnArgs& a, cudaStream_t st, int* launches) {
  if (a.d == 128)
    return a.causal ? launch_attn_t<128, true, PV>(a, st, launches)
                    : launch_attn_t<128, false, PV>(a, st, launches);
  return a.causal ? launch_attn_t<64, true, PV>(a, st, launches)
                  : launch_attn_t<64, false, PV>(a, st, launches);
}

cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st, int* launches) {
  if (a.pv_fp8) return launch_attn_pv<kPvFp8>(a, st, launches);
  return a.pv_f16_accum ? launch_attn_pv<kPvF16Acc>(a, st, launches)
                        : launch_attn_pv<kPvF32>(a, st, launches);
}

// One warp waits on an mbarrier that nothing ever completes, through the
// same bounded wait the attention kernel uses; after limit_ns the wait gives
// up, raises the CTA's abort flag and records site 99 in the status word.
__global__ void bounded_wait_probe_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncwarp();
  warp_wait(&bar, 0, &abort_flag, 99, limit_ns);
}

cudaError_t launch_wait_probe(int limit_ms, cudaStream_t st) {
  bounded_wait_probe_kernel<<<1, 32, 0, st>>>((uint64_t)limit_ms * 1000000ull);
  return cudaGetLastError();
}

cudaError_t device_status_address(int** p) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(p), g_device_status);
}

cudaError_t read_and_clear_device_status(int* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_device_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
}

}  // namespace sage
