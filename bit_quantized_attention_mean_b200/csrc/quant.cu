// quant.cu -- K smoothing and per-block INT8 quantization of Q and K for
// sm_100a (SageAttention article, method section: "对 K 进行平滑处理" and
// "对 Q, K 进行分块 INT8 量化").
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
//     Pass 2 re-reads its rows (from L2), subtracts the mean and quantizes
//     its 64-row blocks, two at a time.
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

__device__ __forceinline__ float block_absmax(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (threadIdx.x < 32) {
    float w = lane < kQuantThreads / 32 ? red[lane] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w = fmaxf(w, __shfl_xor_sync(0xffffffffu, w, o));
    if (lane == 0) red[8] = w;
  }
  __syncthreads();
  const float a = red[8];
  __syncthreads();  // red[] may be reused by the next block
  return a;
}

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

// rne(fl32(x * r)) clamped to [-127, 127], as an int.  The rounding adds
// 1.5 * 2^23 in fp32 (the FADD itself rounds to the nearest integer, ties to
// even, exactly as cvt.rni would for |x * r| < 2^22) and reads the integer
// back from the low mantissa bits; this keeps the conversion off the
// transcendental/conversion unit.
__device__ __forceinline__ int quant_one(float x, float r) {
  const float y = __fmul_rn(x, r);
  const float big = __fadd_rn(y, 12582912.f);
  const int t = __float_as_int(big) - 0x4B400000;
  return max(-127, min(127, t));
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

// Smoothed (for K) fp32 values of one 16-byte vector.
template <bool SMOOTH>
__device__ __forceinline__ void values8(const uint4& raw, const float (&m)[8], float (&x)[8]) {
  unpack8(raw, x);
  if (SMOOTH) {
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = __fsub_rn(x[e], m[e]);
  }
}

// Quantizes one block of `rows` x D fp16 values (row-major) into int8 and
// returns its scale fl32(amax/127).  For K, `m` holds this thread's 8
// channel means (the same channels for every vector of the thread).
template <int D, int ROWS_MAX, bool SMOOTH>
__device__ __forceinline__ float quant_block(const __half* __restrict__ src, int8_t* __restrict__ dst,
                                             int rows, const float (&m)[8], float* red) {
  constexpr int TPR = D / 8;                           // 16-byte vectors per row
  constexpr int VPT = ROWS_MAX * TPR / kQuantThreads;  // vectors per thread
  static_assert(VPT >= 1 && kQuantThreads % TPR == 0, "bad block shape");
  const int nvec = rows * TPR;
  const int tid = threadIdx.x;
  uint4 raw[VPT];
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int idx = tid + v * kQuantThreads;
    raw[v] = idx < nvec ? __ldcs(reinterpret_cast<const uint4*>(src) + idx) : make_uint4(0, 0, 0, 0);
  }
  float amax = 0.f;
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    if (tid + v * kQuantThreads < nvec) {  // padding rows are not in the block
      float x[8];
      values8<SMOOTH>(raw[v], m, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[e]));
    }
  }
  const float a = block_absmax(amax, red);
  const float r = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int idx = tid + v * kQuantThreads;
    if (idx < nvec) {
      float x[8];
      values8<SMOOTH>(raw[v], m, x);
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) lo |= (uint32_t)(quant_one(x[e], r) & 0xff) << (8 * e);
#pragma unroll
      for (int e = 0; e < 4; ++e) hi |= (uint32_t)(quant_one(x[4 + e], r) & 0xff) << (8 * e);
      __stcs(reinterpret_cast<uint2*>(dst) + idx, make_uint2(lo, hi));
    }
  }
  return a > 0.f ? __fdiv_rn(a, 127.f) : 0.f;
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
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) lo |= (uint32_t)(quant_one(x[e], r) & 0xff) << (8 * e);
#pragma unroll
        for (int e = 0; e < 4; ++e) hi |= (uint32_t)(quant_one(x[4 + e], r) & 0xff) << (8 * e);
        __stcs(dst + idx, make_uint2(lo, hi));
      }
    }
    if (tid == 0 && nvec[b] > 0) ks[kb + b] = a > 0.f ? __fdiv_rn(a, 127.f) : 0.f;
  }
}

// ------------------------------------------------------------- kernel

template <int D>
__global__ void __launch_bounds__(kQuantThreads)
quant_qk_kernel(const __half* __restrict__ q, const __half* __restrict__ k,
                int8_t* __restrict__ q_i8, int8_t* __restrict__ k_i8,
                float* __restrict__ q_scale, float* __restrict__ k_scale,
                float* __restrict__ k_mean, int BHkv, int Lq, int Lk, int nqb, int nkb,
                int kb_per_cta, int n_k_ctas, int n_q_blocks, float c) {
  constexpr int TPR = D / 8;
  constexpr int RPP = kQuantThreads / TPR;  // rows per pass of the column sums
  __shared__ float red[32];
  __shared__ long long part[D];   // this CTA's exact column sums (units of 2^-24)
  __shared__ long long rsum[RPP * D > 0 ? RPP * D : 1];
  __shared__ float mean[D];
  const int tid = threadIdx.x;
  const float no_mean[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};

  if ((int)blockIdx.x >= n_k_ctas) {
    // ------------------------------------------------------------ Q block
    const int blk = blockIdx.x - n_k_ctas;
    if (blk >= n_q_blocks) return;  // padding CTA of the last cluster
    const int bh = blk / nqb, qb = blk - bh * nqb;
    const int r0 = qb * SAGE_Q_BLOCK_ROWS;
    const size_t off = ((size_t)bh * Lq + r0) * D;
    const float s = quant_block<D, SAGE_Q_BLOCK_ROWS, false>(
        q + off, q_i8 + off, min(SAGE_Q_BLOCK_ROWS, Lq - r0), no_mean, red);
    if (tid == 0) q_scale[blk] = __fmul_rn(s, c);
    return;
  }

  // -------------------------------------------------------------- K head
  cg::cluster_group cluster = cg::this_cluster();
  const int ncl = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int bhk = blockIdx.x / ncl;
  const int kb0 = min(nkb, rank * kb_per_cta), kb1 = min(nkb, kb0 + kb_per_cta);
  const int t0 = kb0 * SAGE_K_BLOCK_ROWS, t1 = min(Lk, kb1 * SAGE_K_BLOCK_ROWS);
  const __half* kh = k + (size_t)bhk * Lk * D;

  // pass 1: exact column sums of rows [t0, t1)
  {
    const int cg8 = tid % TPR, rr = tid / TPR;
    const uint4* base = reinterpret_cast<const uint4*>(kh) + cg8;
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll 8
    for (int t = t0 + rr; t < t1; t += RPP) {
      float x[8];
      unpack8(__ldg(base + (size_t)t * TPR), x);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += (double)x[e];
    }
    // fp16 values are multiples of 2^-24 below 2^16: each double sum of at
    // most 2^13 of them is exact, and so is its conversion to int64
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
    const double mu = __ddiv_rn(__dmul_rn(__ll2double_rn(s), 0x1p-24), (double)Lk);
    mean[ch] = __double2float_rn(mu);
    if (rank == 0) k_mean[(size_t)bhk * D + ch] = mean[ch];
  }
  cluster.sync();  // no CTA leaves (or reuses part[]) while others read it

  // pass 2: smooth and quantize this CTA's K blocks
  float m8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m8[e] = mean[(tid % TPR) * 8 + e];
  for (int kb = kb0; kb < kb1; kb += 2)
    quant_k_blocks<D, 2>(k + (size_t)bhk * Lk * D, k_i8 + (size_t)bhk * Lk * D,
                         k_scale + (size_t)bhk * nkb, kb, kb1, Lk, m8, red);
}

// ------------------------------------------------------------- launcher

size_t quant_workspace_bytes(int, int, int, int) { return 0; }

template <int D>
static cudaError_t launch_quant_d(const QuantArgs& a, cudaStream_t st, int* launches) {
  const int BH = a.B * a.H, BHkv = a.B * a.Hkv;
  const int nqb = (a.Lq + SAGE_Q_BLOCK_ROWS - 1) / SAGE_Q_BLOCK_ROWS;
  const int nkb = (a.Lk + SAGE_K_BLOCK_ROWS - 1) / SAGE_K_BLOCK_ROWS;
  auto kern = quant_qk_kernel<D>;
  // few heads: wider clusters so the K work spreads over more SMs
  int cl = kCluster;
  if ((long long)BHkv * kCluster < 256 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess)
    cl = 16;
  const int kb_per_cta = (nkb + cl - 1) / cl;
  // a CTA sums at most kb_per_cta * 64 rows; each thread at most 1/RPP of them
  if ((long long)kb_per_cta * SAGE_K_BLOCK_ROWS / (kQuantThreads / (D / 8)) > 8192)
    return cudaErrorInvalidValue;
  const long long n_k_ctas = (long long)BHkv * cl;
  const long long n_q_blocks = (long long)BH * nqb;
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
                                     (int)n_k_ctas, (int)n_q_blocks, a.c);
  *launches += 1;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_quant(const QuantArgs& a, cudaStream_t st, int* launches) {
  return a.d == 128 ? launch_quant_d<128>(a, st, launches) : launch_quant_d<64>(a, st, launches);
}

}  // namespace sage
