// quant.cu -- K smoothing and per-block INT8 quantization of Q and K for
// sm_100a (SageAttention article, method section: the K smoothing step and
// the per-block INT8 quantization step).
//
// One launch, HBM-bound.  The grid is made of thread-block clusters of
// kCluster CTAs (16 when there are few kv heads, so the K work still spreads
// over the chip):
//   * K clusters (one per batch and kv head): CTA r of the cluster owns a
//     range of whole 64-row K blocks.  Pass 1 sums its rows per channel
//     exactly (fp16 values accumulated in double, at most 2^13 terms per
//     thread, then int64 counts of 2^-24); the cluster then adds the
//     kCluster partial sums through distributed shared memory in a fixed
//     order, so every CTA holds the same exact mean (rank 0 stores it).
//     At d = 64 pass 1 also keeps each block's per-channel fp16 minimum and
//     maximum: rounding is monotonic, so with the mean known they give the
//     block's abs-max of fl32(K - mean) exactly, and pass 2 re-reads the rows
//     as one barrier-free stream (subtract, scale, round, store).  Otherwise
//     (d = 128, or more blocks than shared memory holds extremes for) pass 2
//     quantizes two blocks at a time, each reduced across the CTA.
//   * Q clusters: every CTA quantizes one 128-row Q block (Q does not depend
//     on the mean, so this overlaps the K work).
//
// Loads are coalesced 16-byte vectors (8 fp16) kept as raw registers; the
// abs-max (warp shuffles, then shared memory across warps) and the rounding
// pass both convert from them, so nothing is read twice within a block.  All
// float operations use explicit IEEE round-to-nearest intrinsics, so the int8
// codes and scales are bit-reproducible.
#include <cooperative_groups.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "sage_internal.h"

namespace cg = cooperative_groups;

namespace sage {

constexpr int kQuantThreads = 256;
constexpr int kCluster = 8;  // CTAs per K head (16 when there are few heads)

// ------------------------------------------------------------- helpers

// Abs-max of NB independent blocks at once (one value per block per thread).
template <int NB>
__device__ __forceinline__ void block_absmax_n(float (&v)[NB], float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[b] = fmaxf(v[b], __shfl_xor_sync(0xffffffffu, v[b], o));
    if (lane == 0) red[b * 8 + warp] = v[b];
  }
  __syncthreads();
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    float a = red[b * 8];
#pragma unroll
    for (int w = 1; w < kQuantThreads / 32; ++w) a = fmaxf(a, red[b * 8 + w]);
    v[b] = a;
  }
  __syncthreads();  // red[] may be reused by the next group of blocks
}

// The int8 codes rne(fl32(x * r)) of 8 values, packed low byte first.  The
// rounding adds 1.5 * 2^23 in fp32: the FADD itself rounds to the nearest
// integer q (ties to even, as cvt.rni would for |x * r| < 2^22), and the sum's
// bit pattern is 0x4B400000 + q, whose low byte is q's two's-complement code.
// No clamp is needed: every caller has |x| <= a and r = fl32(127 / a), so
// |fl32(x * r)| <= 127 (1 + 2^-24)^2 < 127.5 and |q| <= 127.
// Scalar IEEE operations throughout: the paired fp32 instructions of sm_100
// were measured to round some exact ties (x = a / 2, fl32(x * r) = 63.5)
// differently from round-half-to-even.
__device__ __forceinline__ uint2 quant8(const float (&x)[8], float r) {
  uint32_t w[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) w[e] = __float_as_uint(__fadd_rn(__fmul_rn(x[e], r), 12582912.f));
  const uint32_t lo = __byte_perm(__byte_perm(w[0], w[1], 0x0040), __byte_perm(w[2], w[3], 0x0040),
                                  0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(w[4], w[5], 0x0040), __byte_perm(w[6], w[7], 0x0040),
                                  0x5410);
  return make_uint2(lo, hi);
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&x)[8]) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(h[e]);
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
}

// fp32 values of one 16-byte vector of fp16, smoothed for K: fl32(float(K) - m).
template <bool SMOOTH>
__device__ __forceinline__ void values8(const uint4& raw, const float (&m)[8], float (&x)[8]) {
  unpack8(raw, x);
  if (SMOOTH) {
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = __fsub_rn(x[e], m[e]);
  }
}

// max |h| over the 8 fp16 values of a 16-byte vector, folded into a running
// (max, min) pair of fp16x2 accumulators (exact: fp16 max/min).
__device__ __forceinline__ void absmax8_h(const uint4& u, __half2& mx, __half2& mn) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    mx = __hmax2(mx, h[e]);
    mn = __hmin2(mn, h[e]);
  }
}

__device__ __forceinline__ float absmax_of(const __half2& mx, const __half2& mn) {
  const float2 a = __half22float2(mx), b = __half22float2(mn);
  return fmaxf(fmaxf(a.x, a.y), fmaxf(-b.x, -b.y));
}

// Quantizes one 128-row Q tile whose quantization blocks are QBR rows
// (QBR = 128, 64, 32 or 1) and writes ceil(rows / QBR) scales, each
// multiplied by c.  Thread t holds, for pass v, row t / TPR + RPP * v (RPP =
// rows per pass), so a block of QBR >= RPP rows is a group of passes reduced
// across the CTA, and a one-row block is a group of TPR adjacent lanes.
template <int D, int QBR>
__device__ __forceinline__ void quant_q_tile(const __half* __restrict__ src, int8_t* __restrict__ dst,
                                             float* __restrict__ qs, int rows, float c, float* red) {
  constexpr int TPR = D / 8;
  constexpr int RPP = kQuantThreads / TPR;
  constexpr int VPT = SAGE_Q_BLOCK_ROWS / RPP;
  static_assert(QBR == 1 || (QBR % RPP == 0 && SAGE_Q_BLOCK_ROWS % QBR == 0), "block rows");
  constexpr int NG = QBR == 1 ? VPT : SAGE_Q_BLOCK_ROWS / QBR;  // scale groups per thread
  const int tid = threadIdx.x;
  const int nvec = rows * TPR;
  uint4 raw[VPT];
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int idx = tid + v * kQuantThreads;
    raw[v] = idx < nvec ? __ldcs(reinterpret_cast<const uint4*>(src) + idx) : make_uint4(0, 0, 0, 0);
  }
  const float no_mean[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float amax[NG];
  {
    __half2 mx[NG], mn[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) mx[g] = mn[g] = __float2half2_rn(0.f);
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int g = QBR == 1 ? v : v / (QBR / RPP);
      // rows past the tile were loaded as zeros: they do not change the max
      absmax8_h(raw[v], mx[g], mn[g]);
    }
#pragma unroll
    for (int g = 0; g < NG; ++g) amax[g] = absmax_of(mx[g], mn[g]);
  }
  if (QBR == 1) {
    // the TPR lanes of one row are adjacent within a warp
#pragma unroll
    for (int g = 0; g < NG; ++g)
#pragma unroll
      for (int o = TPR / 2; o > 0; o >>= 1)
        amax[g] = fmaxf(amax[g], __shfl_xor_sync(0xffffffffu, amax[g], o));
  } else {
    block_absmax_n<NG>(amax, red);
  }
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int idx = tid + v * kQuantThreads;
    const int g = QBR == 1 ? v : v / (QBR / RPP);
    const float a = amax[g];
    const float r = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
    if (idx < nvec) {
      float x[8];
      values8<false>(raw[v], no_mean, x);
      __stcs(reinterpret_cast<uint2*>(dst) + idx, quant8(x, r));
    }
    // one thread per block writes its scale
    const int row = idx / TPR;
    const bool writer = QBR == 1 ? (tid % TPR == 0) : (tid == 0 && v % (QBR / RPP) == 0);
    if (writer && row < rows)
      qs[QBR == 1 ? row : row / QBR] = __fmul_rn(a > 0.f ? __fdiv_rn(a, 127.f) : 0.f, c);
  }
}

// Smooths and quantizes NB consecutive K blocks [kb, kb+NB) of one head
// (rows beyond Lk are padding; blocks at or beyond kb_end are skipped).
template <int D, int NB>
__device__ __forceinline__ void quant_k_blocks(const __half* __restrict__ kh, int8_t* __restrict__ kq,
                                               float* __restrict__ ks, int kb, int kb_end, int Lk,
                                               const float (&m)[8], float* red) {
  constexpr int TPR = D / 8;
  constexpr int VPT = SAGE_K_BLOCK_ROWS * TPR / kQuantThreads;
  const int tid = threadIdx.x;
  uint4 raw[NB][VPT];
  int nvec[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const int r0 = (kb + b) * SAGE_K_BLOCK_ROWS;
    nvec[b] = kb + b < kb_end ? min(SAGE_K_BLOCK_ROWS, Lk - r0) * TPR : 0;
    const uint4* src = reinterpret_cast<const uint4*>(kh + (size_t)r0 * D);
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int idx = tid + v * kQuantThreads;
      raw[b][v] = idx < nvec[b] ? __ldcs(src + idx) : make_uint4(0, 0, 0, 0);
    }
  }
  float amax[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    amax[b] = 0.f;
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      if (tid + v * kQuantThreads < nvec[b]) {
        float x[8];
        values8<true>(raw[b][v], m, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax[b] = fmaxf(amax[b], fabsf(x[e]));
      }
    }
  }
  block_absmax_n<NB>(amax, red);
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const float a = amax[b];
    const float r = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
    uint2* dst = reinterpret_cast<uint2*>(kq + (size_t)(kb + b) * SAGE_K_BLOCK_ROWS * D);
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int idx = tid + v * kQuantThreads;
      if (idx < nvec[b]) {
        float x[8];
        values8<true>(raw[b][v], m, x);
        __stcs(dst + idx, quant8(x, r));
      }
    }
    if (tid == 0 && nvec[b] > 0) ks[kb + b] = a > 0.f ? __fdiv_rn(a, 127.f) : 0.f;
  }
}

// ------------------------------------------------------------- kernel

template <int D, int QBR>
__global__ void __launch_bounds__(kQuantThreads, 4)
quant_qk_kernel(const __half* __restrict__ q, const __half* __restrict__ k,
                int8_t* __restrict__ q_i8, int8_t* __restrict__ k_i8,
                float* __restrict__ q_scale, float* __restrict__ k_scale,
                float* __restrict__ k_mean, int BHkv, int Lq, int Lk, int nqb, int nkb,
                int kb_per_cta, int n_k_ctas, int n_q_blocks, float c,
                const int* __restrict__ seqlens_q, const int* __restrict__ seqlens_k, int H,
                int Hkv) {
  constexpr int TPR = D / 8;
  constexpr int RPP = kQuantThreads / TPR;  // rows per pass of the column sums
  __shared__ float red[32];
  __shared__ long long part[D];   // this CTA's exact column sums (units of 2^-24)
  __shared__ long long rsum[RPP * D > 0 ? RPP * D : 1];
  __shared__ float mean[D];
  // per-block channel max and min of K, and 127 / abs-max (d = 64 path)
  __shared__ __half2 kext[D == 64 ? 4096 : 1];
  __shared__ float kr[D == 64 ? 4096 / D : 1];
  const int tid = threadIdx.x;

  if ((int)blockIdx.x >= n_k_ctas) {
    // ------------------------------------------------------------ Q block
    const int blk = blockIdx.x - n_k_ctas;
    if (blk >= n_q_blocks) return;  // padding CTA of the last cluster
    const int bh = blk / nqb, qb = blk - bh * nqb;
    const int r0 = qb * SAGE_Q_BLOCK_ROWS;
    // rows of this head: all Lq, or the entry's own count in a padded batch
    const int Lqb = seqlens_q ? min(max(__ldg(seqlens_q + bh / H), 0), Lq) : Lq;
    if (r0 >= Lqb) return;  // padding rows only
    const size_t off = ((size_t)bh * Lq + r0) * D;
    const int nqs = (Lq + QBR - 1) / QBR;  // scales per head
    quant_q_tile<D, QBR>(q + off, q_i8 + off, q_scale + (size_t)bh * nqs + r0 / QBR,
                         min(SAGE_Q_BLOCK_ROWS, Lqb - r0), c, red);
    return;
  }

  // -------------------------------------------------------------- K head
  cg::cluster_group cluster = cg::this_cluster();
  const int ncl = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int bhk = blockIdx.x / ncl;
  // keys of this head: all Lk, or the entry's own count in a padded batch
  const int Lkb = seqlens_k ? min(max(__ldg(seqlens_k + bhk / Hkv), 0), Lk) : Lk;
  const int nkb_b = (Lkb + SAGE_K_BLOCK_ROWS - 1) / SAGE_K_BLOCK_ROWS;
  const int kb0 = min(nkb_b, rank * kb_per_cta), kb1 = min(nkb_b, kb0 + kb_per_cta);
  const int t0 = kb0 * SAGE_K_BLOCK_ROWS, t1 = min(Lkb, kb1 * SAGE_K_BLOCK_ROWS);
  const __half* kh = k + (size_t)bhk * Lk * D;

  // Per-block channel extremes, kept when this CTA's blocks fit in kFastBlocks:
  // fl32 rounding is monotonic, so over a block the largest |fl32(k - m_c)| of
  // channel c is taken at that channel's smallest or largest k.  Once the mean
  // is known the block abs-max (and so the block scale) follows exactly, and
  // the second pass needs no reduction over the rows it re-reads.
  // Used at d = 64, where it measured 8 % faster; at d = 128 it measured
  // 1-7 % slower (its extra registers spill in a kernel whose register budget
  // the Q tiles share).
  constexpr bool kExtremes = D == 64;
  constexpr int kFastBlocks = kExtremes ? 4096 / D : 0;
  const int nb = kb1 - kb0;
  const bool fast = kExtremes && nb <= kFastBlocks;
  constexpr int R = 32 / TPR;  // rows per warp-wide load (each lane: one 16-byte vector)
  const int warp = tid >> 5, lane = tid & 31;
  const int sub = lane / TPR, cg8 = lane % TPR;

  // pass 1: exact column sums of rows [t0, t1).  Lane (sub, cg8) of warp w
  // is row class rr = w * R + sub = tid / TPR for the channels of cg8.
  {
    const uint4* base = reinterpret_cast<const uint4*>(kh) + cg8;
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;
    auto add8 = [&](const uint4& u) {
      const unsigned short* h = reinterpret_cast<const unsigned short*>(&u);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        double x;  // fp16 -> fp64 is exact
        asm("cvt.f64.f16 %0, %1;" : "=d"(x) : "h"(h[e]));
        acc[e] += x;
      }
    };
    if constexpr (!kExtremes) {
      // row class rr takes every RPP-th row
#pragma unroll 8
      for (int t = t0 + tid / TPR; t < t1; t += RPP) add8(__ldg(base + (size_t)t * TPR));
    } else {
      // warp w takes whole blocks w, w + 8, ... and their channel extremes
      for (int bl = warp; bl < nb; bl += kQuantThreads / 32) {
        const int r0 = t0 + bl * SAGE_K_BLOCK_ROWS;
        const int r1 = min(t1, r0 + SAGE_K_BLOCK_ROWS);
        __half2 mx[4], mn[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          mx[e] = __float2half2_rn(-INFINITY);
          mn[e] = __float2half2_rn(INFINITY);
        }
#pragma unroll 8
        for (int t = r0 + sub; t < r1; t += R) {
          const uint4 u = __ldg(base + (size_t)t * TPR);
          add8(u);
          const __half2* h2 = reinterpret_cast<const __half2*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            mx[e] = __hmax2(mx[e], h2[e]);
            mn[e] = __hmin2(mn[e], h2[e]);
          }
        }
        if (fast) {
          // the R lanes holding the same channels are TPR apart
#pragma unroll
          for (int o = TPR; o < 32; o <<= 1)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              mx[e] = __hmax2(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], o));
              mn[e] = __hmin2(mn[e], __shfl_xor_sync(0xffffffffu, mn[e], o));
            }
          if (sub == 0) {
            // block bl: per 8-channel group, 4 fp16x2 maxima then 4 minima
            __half2* dst = kext + (size_t)bl * D + cg8 * 8;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              dst[e] = mx[e];
              dst[4 + e] = mn[e];
            }
          }
        }
      }
    }
    // fp16 values are multiples of 2^-24 below 2^16: each double sum of at
    // most 2^13 of them is exact, and so is its conversion to int64
    const int rr = warp * R + sub;  // one of RPP row classes
#pragma unroll
    for (int e = 0; e < 8; ++e) rsum[rr * D + cg8 * 8 + e] = (long long)(acc[e] * 16777216.0);
    __syncthreads();
    for (int ch = tid; ch < D; ch += kQuantThreads) {
      long long s = 0;
      for (int i = 0; i < RPP; ++i) s += rsum[i * D + ch];
      part[ch] = s;
    }
  }
  cluster.sync();  // every CTA's partial sums are visible cluster-wide
  for (int ch = tid; ch < D; ch += kQuantThreads) {
    long long s = 0;
    for (int r = 0; r < ncl; ++r) s += *cluster.map_shared_rank(&part[ch], r);
    const double mu = Lkb > 0 ? __ddiv_rn(__dmul_rn(__ll2double_rn(s), 0x1p-24), (double)Lkb) : 0.0;
    mean[ch] = __double2float_rn(mu);
    if (rank == 0) k_mean[(size_t)bhk * D + ch] = mean[ch];
  }
  cluster.sync();  // no CTA leaves (or reuses part[]) while others read it

  float m8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m8[e] = mean[(tid % TPR) * 8 + e];
  if (!fast) {
    // pass 2 (d = 128, or more blocks than the extremes cover): re-read,
    // smooth and quantize two blocks at a time
    for (int kb = kb0; kb < kb1; kb += 2)
      quant_k_blocks<D, 2>(k + (size_t)bhk * Lk * D, k_i8 + (size_t)bhk * Lk * D,
                           k_scale + (size_t)bhk * nkb, kb, kb1, Lkb, m8, red);
    return;
  }

  // block scales from the extremes: 8 lanes per block, D/8 channels each; the
  // loop bound is warp-uniform so every lane reaches the shuffles
  {
    constexpr int CPL = D / 8;
    for (int base = warp * 4; base < nb; base += kQuantThreads / 8) {
      const int bl = base + lane / 8;
      float a = 0.f;
      if (bl < nb) {
        const __half* ext = reinterpret_cast<const __half*>(kext + (size_t)bl * D);
        const int c0 = (lane % 8) * CPL;
#pragma unroll 8
        for (int c = c0; c < c0 + CPL; ++c) {
          // channel c: its 8-channel group's maxima, then its minima
          const int g = (c >> 3) * 16 + (c & 7);
          const float hi = __half2float(ext[g]), lo = __half2float(ext[g + 8]);
          a = fmaxf(a, fabsf(__fsub_rn(hi, mean[c])));
          a = fmaxf(a, fabsf(__fsub_rn(lo, mean[c])));
        }
      }
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      if (bl < nb && lane % 8 == 0) {
        kr[bl] = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
        k_scale[(size_t)bhk * nkb + kb0 + bl] = a > 0.f ? __fdiv_rn(a, 127.f) : 0.f;
      }
    }
  }
  __syncthreads();

  // pass 2: one stream over the rows [t0, t1): smooth, quantize, store
  {
    const int nvec = (t1 - t0) * TPR;
    const uint4* src = reinterpret_cast<const uint4*>(kh + (size_t)t0 * D);
    uint2* dst = reinterpret_cast<uint2*>(k_i8 + ((size_t)bhk * Lk + t0) * D);
    constexpr int U = 8;
    for (int i0 = tid; i0 < nvec; i0 += U * kQuantThreads) {
      uint4 raw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int idx = i0 + u * kQuantThreads;
        raw[u] = idx < nvec ? __ldcs(src + idx) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int idx = i0 + u * kQuantThreads;
        if (idx < nvec) {
          float x[8];
          values8<true>(raw[u], m8, x);
          __stcs(dst + idx, quant8(x, kr[idx / (SAGE_K_BLOCK_ROWS * TPR)]));
        }
      }
    }
  }
}

// ------------------------------------------------------------- launcher

template <int D, int QBR>
static cudaError_t launch_quant_d(const QuantArgs& a, cudaStream_t st, int* launches) {
  const int BH = a.B * a.H, BHkv = a.B * a.Hkv;
  const int nqb = (a.Lq + SAGE_Q_BLOCK_ROWS - 1) / SAGE_Q_BLOCK_ROWS;
  const int nkb = (a.Lk + SAGE_K_BLOCK_ROWS - 1) / SAGE_K_BLOCK_ROWS;
  auto kern = quant_qk_kernel<D, QBR>;
  // few heads: wider clusters so the K work spreads over more SMs
  int cl = kCluster;
  if ((long long)BHkv * kCluster < 256 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess)
    cl = 16;
  const int kb_per_cta = (nkb + cl - 1) / cl;
  // a CTA sums kb_per_cta blocks of 64 rows, each warp every 8th block and
  // each lane 1/R of a block's rows (R = 32 / (D / 8)): at most 2^13 exact
  // double sums per lane; the entry points refuse Lk above
  // SAGE_MAX_LK (2^20), which keeps this bound for every cluster width and d
  if ((long long)(kb_per_cta + 7) / 8 * (SAGE_K_BLOCK_ROWS / (32 / (D / 8))) > 8192)
    return cudaErrorInvalidValue;
  const long long n_k_ctas = (long long)BHkv * cl;
  const long long n_q_blocks = a.skip_q ? 0 : (long long)BH * nqb;
  const long long n_q_ctas = (n_q_blocks + cl - 1) / cl * cl;
  if (n_k_ctas + n_q_ctas > 0x7fffffffLL) return cudaErrorInvalidConfiguration;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(n_k_ctas + n_q_ctas), 1, 1);
  cfg.blockDim = dim3(kQuantThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a.q, a.k, a.q_i8, a.k_i8, a.q_scale, a.k_scale,
                                     a.k_mean, BHkv, a.Lq, a.Lk, nqb, nkb, kb_per_cta,
                                     (int)n_k_ctas, (int)n_q_blocks, a.c, a.seqlens_q,
                                     a.seqlens_k, a.H, a.Hkv);
  *launches += 1;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_quant_qbr(const QuantArgs& a, cudaStream_t st, int* launches) {
  switch (a.q_block_rows) {
    case 128: return launch_quant_d<D, 128>(a, st, launches);
    case 64: return launch_quant_d<D, 64>(a, st, launches);
    case 32: return launch_quant_d<D, 32>(a, st, launches);
    case 1: return launch_quant_d<D, 1>(a, st, launches);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_quant(const QuantArgs& a, cudaStream_t st, int* launches) {
  return a.d == 128 ? launch_quant_qbr<128>(a, st, launches)
                    : launch_quant_qbr<64>(a, st, launches);
}

}  // namespace sage
