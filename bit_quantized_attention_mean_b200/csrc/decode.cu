// decode.cu -- 8-bit quantized attention of a few query tokens against a long
// key sequence (decoding against a KV cache), for sm_100a.
//
// Same arithmetic as the forward kernel (SageAttention article, method
// section: INT8 Q K^T with an INT32 accumulator, dequantization by
// q_scale * k_scale, base-2 online softmax, FP16 P V), laid out for Lq << Lk,
// where the work is bound by reading K and V once from HBM:
//   * the H / Hkv query heads that share a kv head ("GQA") are packed into
//     one 128-row tile, row g * Lq + i for head g of the group and query i,
//     so each K/V tile is read once per group instead of once per head;
//   * the keys are split into nsplit ranges handled by different CTAs
//     (grid = B * Hkv * nsplit, about two CTAs per SM), each producing an
//     unnormalized partial output with its running max and sum; a second
//     kernel merges the splits (skipped when nsplit = 1);
//   * softmax warps whose 32 rows are all padding only keep the barrier
//     protocol going, so a tile with few real rows costs little arithmetic;
//   * optionally each batch entry has its own number of keys (variable-length
//     caches in one padded buffer): splits past an entry's length are empty;
//   * optionally the cache is paged: 64-key pages (one K quantization block
//     each) of all kv heads, found through a per-entry block table.
// Warp roles, tensor-memory layout, barriers and the bounded waits are those
// of the forward kernel: warp 4 issues TMA loads, one thread of warp 5 the
// tcgen05 MMAs, warps 0-3 own the rows.
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

constexpr int kDecRows = 128;  // packed query rows per tile
constexpr int kDecKeys = 64;   // keys per tile (= K quantization block)

template <int D>
struct DecCfg {
  static constexpr int STAGES = 3;
  static constexpr int Q_BYTES = kDecRows * D;      // int8
  static constexpr int K_BYTES = kDecKeys * D;      // int8, per stage
  static constexpr int V_BYTES = kDecKeys * D * 2;  // fp16, per stage
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * K_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * V_BYTES;
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
  // at most two CTAs per SM: tensor memory holds two 256-column allocations
  static constexpr int SMEM_BYTES = (USED + 1024) > 80 * 1024 ? (USED + 1024) : 80 * 1024;
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t S_COL = 0;  // buffer b at S_COL + 64 * b
  static constexpr uint32_t O_COL = 128;
  static constexpr uint32_t QK_SWIZZLE = D == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t QK_SBO = 8 * D;
  static_assert(Q_BYTES % 1024 == 0 && K_BYTES % 1024 == 0 && V_BYTES % 1024 == 0,
                "tiles must stay 1024-byte aligned");
};

__device__ __forceinline__ bool dec_warp_wait(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag, int* status, int site) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status, site);
  return __all_sync(0xffffffffu, ok);
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(192, 2)
sage_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ q_scale,
                   const float* __restrict__ k_scale, __half* __restrict__ out,
                   float* __restrict__ o_part, float2* __restrict__ ml_part,
                   const int* __restrict__ seqlens, const int* __restrict__ block_table,
                   int max_blocks, int num_pages, int H, int Hkv, int G, int Lq, int Lk,
                   int nsplit, int split_tiles, int qbr, int* status) {
  using C = DecCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bhk = blockIdx.x / nsplit, sp = blockIdx.x - bhk * nsplit;
  const int b = bhk / Hkv, hkv = bhk - b * Hkv;
  const int rows = G * Lq;  // packed rows in use
  const int nkb = (Lk + kDecKeys - 1) / kDecKeys;  // k_scale row length (the cache's)
  // keys of this batch entry: all Lk, or its own length in a shared cache
  const int Lb = seqlens ? min(max(__ldg(seqlens + b), 0), Lk) : Lk;
  const int t0 = sp * split_tiles;
  const int nkt = max(0, min((Lb + kDecKeys - 1) / kDecKeys, t0 + split_tiles) - t0);
  // Paged caches: key tile t of entry b is page block_table[b][t] (64 keys of
  // every kv head); its K/V rows are at TMA coordinate z = page * Hkv + hkv
  // and its k_scale at [page][hkv].  Pages outside [0, num_pages) are clamped.
  auto page_of = [&](int t) {
    return min(max(__ldg(block_table + (size_t)b * max_blocks + t), 0), num_pages - 1);
  };

  if (tid == 0) {
    for (int i = 0; i < C::NUM_BARS; ++i)
      mbar_init(&bars[i], (i == C::B_P_FULL || i == C::B_P_FULL + 1) ? 128u : 1u);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  // padding rows of the Q tile hold zeros (their scores are then 0)
  if (tid < kDecRows && tid >= rows) {
    uint4* row = reinterpret_cast<uint4*>(smem + C::OFF_Q + tid * D);
#pragma unroll
    for (int c = 0; c < D / 16; ++c) row[c] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
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
      const uint64_t stream = l2_policy_evict_first();  // K/V are read once
      mbar_arrive_expect_tx(&bars[C::B_Q_FULL], (uint32_t)(rows * D));
      tma_load_4d(smem + C::OFF_Q, &tm_q, &bars[C::B_Q_FULL], 0, 0, 0, bhk);
      int issued = 0;
      for (int j = 0; j < nkt; ++j) {
        const int s = j % C::STAGES;
        if (j >= C::STAGES &&
            !mbar_wait(&bars[C::B_KV_EMPTY + s], ((j / C::STAGES) - 1) & 1, abort_flag, status, 31))
          break;
        mbar_arrive_expect_tx(&bars[C::B_K_FULL + s], C::K_BYTES);
        int ky = (t0 + j) * kDecKeys, kz = bhk;
        if (block_table) {
          ky = 0;
          kz = page_of(t0 + j) * Hkv + hkv;
        }
        tma_load_3d_hint(smem + C::OFF_K + s * C::K_BYTES, &tm_k, &bars[C::B_K_FULL + s], 0, ky,
                         kz, stream);
        mbar_arrive_expect_tx(&bars[C::B_V_FULL + s], C::V_BYTES);
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc)
          tma_load_3d_hint(smem + C::OFF_V + s * C::V_BYTES + cc * (kDecKeys * 128), &tm_v,
                           &bars[C::B_V_FULL + s], cc * 64, ky, kz, stream);
        issued = j + 1;
      }
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
      constexpr uint32_t idesc_qk = make_idesc_i8(kDecRows, kDecKeys);
      constexpr uint32_t idesc_pv = make_idesc_f16(kDecRows, D, /*b_mn_major=*/true);
      const uint32_t sQ = smem_u32(smem + C::OFF_Q);
      auto issue_pv = [&](int jj) -> bool {
        const int bb = jj & 1, ss = jj % C::STAGES;
        if (!mbar_wait(&bars[C::B_P_FULL + bb], (jj >> 1) & 1, abort_flag, status, 32)) return false;
        if (!mbar_wait(&bars[C::B_V_FULL + ss], (jj / C::STAGES) & 1, abort_flag, status, 33))
          return false;
        tc_fence_after_sync();
        const uint32_t sV = smem_u32(smem + C::OFF_V + ss * C::V_BYTES);
        const uint32_t p_tmem = tmem + C::S_COL + 64u * bb;
#pragma unroll
        for (int kk = 0; kk < kDecKeys / 16; ++kk) {
          const uint64_t bdesc =
              make_smem_desc(sV + kk * 16 * 128, kDecKeys * 128, 1024, kSwizzle128B);
          umma_f16_ts(tmem + C::O_COL, p_tmem + kk * 8, bdesc, idesc_pv,
                      (jj > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars[C::B_KV_EMPTY + ss]);
        umma_commit(&bars[C::B_O_DONE]);
        return true;
      };
      bool ok = mbar_wait(&bars[C::B_Q_FULL], 0, abort_flag, status, 34);
      if (ok) {
        tc_fence_after_sync();
        for (int j = 0; j < nkt; ++j) {
          const int s = j % C::STAGES, bb = j & 1;
          if (!mbar_wait(&bars[C::B_K_FULL + s], (j / C::STAGES) & 1, abort_flag, status, 35)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sK = smem_u32(smem + C::OFF_K + s * C::K_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
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
      umma_commit(&bars[C::B_TEARDOWN]);
      mbar_wait_drain(&bars[C::B_TEARDOWN], 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    const int row = tid;
    const bool real = row < rows;
    const bool idle = warp * 32 >= rows;  // every row of this warp is padding
    const int g = real ? row / Lq : 0, i = real ? row - g * Lq : 0;
    const int bh = b * H + hkv * G + g;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int nqs = (Lq + qbr - 1) / qbr;
    const float sq = real ? __ldg(q_scale + (size_t)bh * nqs + i / qbr) : 0.f;
    auto kscale = [&](int t) {
      return __ldg(block_table ? k_scale + (size_t)page_of(t) * Hkv + hkv
                               : k_scale + (size_t)bhk * nkb + t);
    };
    const int diag = i + (Lb - Lq) + 1;  // keys [0, diag) visible to this row
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    float ck = nkt > 0 ? kscale(t0) : 0.f;
    for (int j = 0; j < nkt; ++j) {
      const int bb = j & 1;
      const float c = __fmul_rn(sq, ck);
      if (j + 1 < nkt) ck = kscale(t0 + j + 1);
      if (!dec_warp_wait(&bars[C::B_S_FULL + bb], (j >> 1) & 1, abort_flag, status, 36)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t s_tmem = tmem + lane_base + C::S_COL + 64u * bb;
      if (!idle) {
        uint32_t s[64];
        tmem_ld64(s_tmem, s);
        const int key0 = (t0 + j) * kDecKeys;
        int vis = real ? Lb - key0 : 0;
        if (CAUSAL) vis = min(vis, diag - key0);
        const bool full = vis >= kDecKeys;
        int mx = INT_MIN;
        if (full) {
#pragma unroll
          for (int k = 0; k < kDecKeys; ++k) mx = max(mx, (int)s[k]);
        } else {
#pragma unroll
          for (int k = 0; k < kDecKeys; ++k) mx = (k < vis) ? max(mx, (int)s[k]) : mx;
        }
        const float mt = vis > 0 ? (float)mx * c : -INFINITY;
        const bool need = mt > m_run + 8.0f;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx(m_run - mt);
          m_run = mt;
        }
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // S_j's commit came after P V_{j-2} was issued: O_DONE is at most
          // one phase behind P V_{j-1}
          if (!dec_warp_wait(&bars[C::B_O_DONE], (j - 1) & 1, abort_flag, status, 37)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_base + C::O_COL + cc * 32, o);
#pragma unroll
            for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
            tmem_st32(tmem + lane_base + C::O_COL + cc * 32, o);
          }
        }
        l_run *= alpha;
        const float moff = m_run == -INFINITY ? 0.f : m_run;
        uint32_t pk[32];
        float lsum = 0.f;
#pragma unroll
        for (int k = 0; k < kDecKeys; k += 2) {
          // |S| <= 127*127*128 < 2^24: the int -> float conversion is exact
          const float x0 = __int2float_rn((int)s[k]);
          const float x1 = __int2float_rn((int)s[k + 1]);
          float p0 = ex2_approx(fmaf(x0, c, -moff));
          float p1 = ex2_approx(fmaf(x1, c, -moff));
          if (!full) {
            p0 = k < vis ? p0 : 0.f;
            p1 = k + 1 < vis ? p1 : 0.f;
          }
          lsum += p0 + p1;
          pk[k >> 1] = pack_half2(p0, p1);
        }
        l_run += lsum;
        tmem_st32(s_tmem, pk);
      }
      tc_fence_before_sync();
      mbar_arrive(&bars[C::B_P_FULL + bb]);
    }
    if (ok && nkt > 0) {
      ok = dec_warp_wait(&bars[C::B_O_FINAL], 0, abort_flag, status, 38);
      tc_fence_after_sync();
    }
    if (ok && !idle) {
      const bool direct = nsplit == 1;
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      __half* orow = out + ((size_t)bh * Lq + i) * D;
      float* prow = o_part + ((size_t)blockIdx.x * rows + row) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        if (nkt > 0) {
          tmem_ld32(tmem + lane_base + C::O_COL + cc * 32, o);
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = 0u;
        }
        if (!real) continue;
        if (direct) {
          uint32_t hv[16];
#pragma unroll
          for (int q = 0; q < 16; ++q)
            hv[q] = pack_half2(__uint_as_float(o[2 * q]) * inv, __uint_as_float(o[2 * q + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
        } else {
          float4* dst = reinterpret_cast<float4*>(prow + cc * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(o[4 * q]), __uint_as_float(o[4 * q + 1]),
                                 __uint_as_float(o[4 * q + 2]), __uint_as_float(o[4 * q + 3]));
        }
      }
      if (real && !direct) ml_part[(size_t)blockIdx.x * rows + row] = make_float2(m_run, l_run);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Merges the key splits of one output row: O = sum_s O_s 2^(m_s - M) /
// sum_s l_s 2^(m_s - M), M = max_s m_s (base-2 running maxima).  One CTA of
// D threads per (batch, head, query) row; thread c owns channel c.
template <int D>
__global__ void __launch_bounds__(D)
sage_decode_combine_kernel(const float* __restrict__ o_part, const float2* __restrict__ ml_part,
                           __half* __restrict__ out, int H, int Hkv, int G, int Lq, int nsplit) {
  const int r = blockIdx.x;  // ((b * H) + h) * Lq + i
  const int i = r % Lq, bh = r / Lq;
  const int b = bh / H, h = bh - b * H;
  const int hkv = h / G, g = h - hkv * G;
  const int rows = G * Lq, row = g * Lq + i;
  const size_t base = (size_t)(b * Hkv + hkv) * nsplit;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, ml_part[(base + s) * rows + row].x);
  float L = 0.f, acc = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < nsplit; ++s) {
      const float2 ml = ml_part[(base + s) * rows + row];
      if (ml.x == -INFINITY) continue;
      const float w = exp2f(ml.x - M);
      L += ml.y * w;
      acc += o_part[((base + s) * rows + row) * D + threadIdx.x] * w;
    }
  }
  out[(size_t)r * D + threadIdx.x] = __float2half_rn(L > 0.f ? acc / L : 0.f);
}

// ------------------------------------------------------------------- host

static PFN_cuTensorMapEncodeTiled_v12000 dec_tensor_map_encoder() {
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

static bool dec_make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esize,
                         int rank, const uint64_t* dims, const uint32_t* box,
                         CUtensorMapSwizzle sw) {
  auto enc = dec_tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t d[4], strides[3];
  cuuint32_t bx[4], estr[4] = {1, 1, 1, 1};
  uint64_t stride = (uint64_t)esize;
  for (int r = 0; r < rank; ++r) {
    d[r] = dims[r];
    bx[r] = box[r];
    if (r > 0) strides[r - 1] = stride;
    stride *= dims[r];
  }
  return enc(map, dt, (cuuint32_t)rank, const_cast<void*>(base), d, strides, bx, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

DecodePlan decode_plan(int B, int H, int Hkv, int Lq, int Lk, int d) {
  DecodePlan p{};
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int nkb = (Lk + kDecKeys - 1) / kDecKeys;
  const long long groups = (long long)B * Hkv;
  // at most two CTAs per SM in one wave: a second, partial wave would leave
  // most of the GPU idle while it runs
  long long want = (2LL * sms) / groups;
  if (want < 1) want = 1;
  if (want > nkb) want = nkb;
  p.split_tiles = (int)((nkb + want - 1) / want);
  p.nsplit = (nkb + p.split_tiles - 1) / p.split_tiles;
  p.rows = (H / Hkv) * Lq;
  const size_t parts = (size_t)groups * p.nsplit * p.rows;
  p.o_bytes = p.nsplit > 1 ? ((parts * d * 4 + 255) & ~(size_t)255) : 0;
  p.ml_bytes = p.nsplit > 1 ? ((parts * 8 + 255) & ~(size_t)255) : 0;
  return p;
}

template <int D, bool CAUSAL>
static cudaError_t launch_decode_t(const DecodeArgs& a, const DecodePlan& p, cudaStream_t st,
                                   int* launches) {
  using C = DecCfg<D>;
  auto kern = sage_decode_kernel<D, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int G = a.H / a.Hkv;
  const CUtensorMapSwizzle qk_sw =
      D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap tq, tk, tv;
  const uint64_t qd[4] = {(uint64_t)D, (uint64_t)a.Lq, (uint64_t)G, (uint64_t)a.B * a.Hkv};
  const uint32_t qb[4] = {(uint32_t)D, (uint32_t)a.Lq, (uint32_t)G, 1u};
  // contiguous cache [B*Hkv, Lk, d]; paged cache [num_pages*Hkv, 64, d]
  const uint64_t kd[3] = {(uint64_t)D, a.block_table ? (uint64_t)kDecKeys : (uint64_t)a.Lk,
                          a.block_table ? (uint64_t)a.num_pages * a.Hkv : (uint64_t)a.B * a.Hkv};
  const uint32_t kb[3] = {(uint32_t)D, (uint32_t)kDecKeys, 1u};
  const uint32_t vb[3] = {64u, (uint32_t)kDecKeys, 1u};
  if (!dec_make_map(&tq, a.q_i8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 4, qd, qb, qk_sw) ||
      !dec_make_map(&tk, a.k_i8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 3, kd, kb, qk_sw) ||
      !dec_make_map(&tv, a.v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, 3, kd, vb,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int* status = nullptr;
  if ((e = device_status_address(&status)) != cudaSuccess) return e;
  const long long grid = (long long)a.B * a.Hkv * p.nsplit;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  kern<<<(unsigned)grid, 192, C::SMEM_BYTES, st>>>(tq, tk, tv, a.q_scale, a.k_scale, a.out,
                                                   a.o_part, a.ml_part, a.seqlens, a.block_table,
                                                   a.max_blocks, a.num_pages, a.H, a.Hkv, G,
                                                   a.Lq, a.Lk,
                                                   p.nsplit, p.split_tiles, a.q_block_rows,
                                                   status);
  *launches += 1;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (p.nsplit > 1) {
    const long long nrows = (long long)a.B * a.H * a.Lq;
    sage_decode_combine_kernel<D><<<(unsigned)nrows, D, 0, st>>>(a.o_part, a.ml_part, a.out, a.H,
                                                                 a.Hkv, G, a.Lq, p.nsplit);
    *launches += 1;
    e = cudaGetLastError();
  }
  return e;
}

cudaError_t launch_decode(const DecodeArgs& a, const DecodePlan& p, cudaStream_t st,
                          int* launches) {
  if (a.d == 128)
    return a.causal ? launch_decode_t<128, true>(a, p, st, launches)
                    : launch_decode_t<128, false>(a, p, st, launches);
  return a.causal ? launch_decode_t<64, true>(a, p, st, launches)
                  : launch_decode_t<64, false>(a, p, st, launches);
}

}  // namespace sage
