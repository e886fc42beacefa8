// quant.cu -- K smoothing and per-block INT8 quantization of Q and K for
// sm_100a (SageAttention article, method section: "对 K 进行平滑处理" and
// "对 Q, K 进行分块 INT8 量化").
//
// Three launches on the caller's stream, all HBM-bound streaming kernels:
//   1. kmean_and_quant_q: CTAs [0, n_chunk_ctas) reduce 256-token chunks of K
//      to exact int64 fixed-point column sums (units of 2^-24); the remaining
//      CTAs quantize one 128-row Q block each (Q does not depend on the mean,
//      so its quantization overlaps the K reduction).
//   2. kmean_finalize: sums the chunk partials in int64 (exact, order free)
//      and writes the fp32 mean per (batch, kv head, channel).
//   3. quant_k: smooths and quantizes one 64-row K block per CTA.
//
// Every load is a coalesced 16-byte vector (8 fp16); a block's rows stay in
// registers between the abs-max reduction (warp shuffles, then shared memory
// across the 8 warps) and the rounding pass, so each element is read from HBM
// once per pass.  All float operations use explicit IEEE round-to-nearest
// intrinsics so the int8 codes and scales are bit-reproducible.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "sage_internal.h"

namespace sage {

constexpr int kQuantThreads = 256;
constexpr int kMeanChunk = 256;  // tokens per K-mean partial

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
  return red[8];
}

__device__ __forceinline__ int quant_one(float x, float r) {
  int t = __float2int_rn(__fmul_rn(x, r));  // round half to even
  return max(-127, min(127, t));
}

__device__ __forceinline__ uint2 quant_pack8(const float (&x)[8], float r) {
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) lo |= (uint32_t)(quant_one(x[e], r) & 0xff) << (8 * e);
#pragma unroll
  for (int e = 0; e < 4; ++e) hi |= (uint32_t)(quant_one(x[4 + e], r) & 0xff) << (8 * e);
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

// Quantizes one block of `rows` x D values (row-major, fp16) into int8 and
// returns the block scale fl32(amax/127).  `mean` (K only) is subtracted per
// channel first.  ROWS_MAX is 128 (Q) or 64 (K).
template <int D, int ROWS_MAX, bool SMOOTH>
__device__ __forceinline__ float quant_block(const __half* __restrict__ src, int8_t* __restrict__ dst,
                                             int rows, const float* __restrict__ mean, float* red) {
  constexpr int TPR = D / 8;                                // 16-byte vectors per row
  constexpr int VPT = ROWS_MAX * TPR / kQuantThreads;       // vectors per thread
  static_assert(VPT >= 1 && kQuantThreads % TPR == 0, "bad block shape");
  const int nvec = rows * TPR;
  const int tid = threadIdx.x;

  float m[8];
  if (SMOOTH) {
    const int ch0 = (tid % TPR) * 8;  // the same channels for every vector of this thread
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = __ldg(mean + ch0 + e);
  }

  float x[VPT][8];
  uint4 raw[VPT];
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int idx = tid + v * kQuantThreads;
    raw[v] = idx < nvec ? __ldg(reinterpret_cast<const uint4*>(src) + idx) : make_uint4(0, 0, 0, 0);
  }
  float amax = 0.f;
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    unpack8(raw[v], x[v]);
    const bool live = tid + v * kQuantThreads < nvec;  // padding rows are not in the block
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float t = SMOOTH ? __fsub_rn(x[v][e], m[e]) : x[v][e];
      x[v][e] = live ? t : 0.f;
      amax = fmaxf(amax, fabsf(x[v][e]));
    }
  }
  const float a = block_absmax(amax, red);
  const float r = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int idx = tid + v * kQuantThreads;
    if (idx < nvec) reinterpret_cast<uint2*>(dst)[idx] = quant_pack8(x[v], r);
  }
  return a > 0.f ? __fdiv_rn(a, 127.f) : 0.f;
}

// ------------------------------------------------------------- kernels

// Exact column sums of one 256-token chunk of K for one (batch, kv head).
// A thread sums at most kMeanChunk / RPP values per channel in double, which
// is exact (fp16 values are multiples of 2^-24 below 2^16 in magnitude, and
// the partial stays below 2^53 units); the result is an int64 count of 2^-24.
template <int D>
__device__ __forceinline__ void kmean_chunk(const __half* __restrict__ k, long long* __restrict__ part,
                                            int Lk, int bhk, int chunk, int nchunks,
                                            long long* red /* [RPP][D] */) {
  constexpr int TPR = D / 8;
  constexpr int RPP = kQuantThreads / TPR;  // rows per pass
  const int tid = threadIdx.x;
  const int cg = tid % TPR, rr = tid / TPR;
  const int t0 = chunk * kMeanChunk;
  const int t1 = min(Lk, t0 + kMeanChunk);
  const uint4* base = reinterpret_cast<const uint4*>(k + (size_t)bhk * Lk * D) + cg;
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll 4
  for (int t = t0 + rr; t < t1; t += RPP) {
    float x[8];
    unpack8(__ldg(base + (size_t)t * TPR), x);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += (double)x[e];
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rr * D + cg * 8 + e] = (long long)(acc[e] * 16777216.0);
  __syncthreads();
  for (int c = tid; c < D; c += kQuantThreads) {
    long long s = 0;
    for (int i = 0; i < RPP; ++i) s += red[i * D + c];
    part[((size_t)bhk * nchunks + chunk) * D + c] = s;
  }
}

template <int D>
__global__ void __launch_bounds__(kQuantThreads)
kmean_and_quant_q_kernel(const __half* __restrict__ q, const __half* __restrict__ k,
                         int8_t* __restrict__ q_i8, float* __restrict__ q_scale,
                         long long* __restrict__ part, int BHkv, int BH, int Lq, int Lk,
                         int nchunks, int nqb, float c) {
  __shared__ float red[16];
  __shared__ long long kred[kQuantThreads / (D / 8) * D];
  const int n_mean = BHkv * nchunks;
  int blk = blockIdx.x;
  if (blk < n_mean) {
    kmean_chunk<D>(k, part, Lk, blk / nchunks, blk % nchunks, nchunks, kred);
    return;
  }
  blk -= n_mean;
  const int bh = blk / nqb, qb = blk - bh * nqb;
  const int r0 = qb * SAGE_Q_BLOCK_ROWS;
  const int rows = min(SAGE_Q_BLOCK_ROWS, Lq - r0);
  const size_t off = ((size_t)bh * Lq + r0) * D;
  const float s = quant_block<D, SAGE_Q_BLOCK_ROWS, false>(q + off, q_i8 + off, rows, nullptr, red);
  if (threadIdx.x == 0) q_scale[blk] = __fmul_rn(s, c);
}

template <int D>
__global__ void kmean_finalize_kernel(const long long* __restrict__ part, float* __restrict__ k_mean,
                                      int Lk, int nchunks) {
  const int bhk = blockIdx.x, c = threadIdx.x;
  long long s = 0;
  for (int i = 0; i < nchunks; ++i) s += part[((size_t)bhk * nchunks + i) * D + c];
  const double mean = __ddiv_rn(__dmul_rn(__ll2double_rn(s), 0x1p-24), (double)Lk);
  k_mean[(size_t)bhk * D + c] = __double2float_rn(mean);
}

template <int D>
__global__ void __launch_bounds__(kQuantThreads)
quant_k_kernel(const __half* __restrict__ k, const float* __restrict__ k_mean,
               int8_t* __restrict__ k_i8, float* __restrict__ k_scale, int Lk, int nkb) {
  __shared__ float red[16];
  const int blk = blockIdx.x;
  const int bhk = blk / nkb, kb = blk - bhk * nkb;
  const int r0 = kb * SAGE_K_BLOCK_ROWS;
  const int rows = min(SAGE_K_BLOCK_ROWS, Lk - r0);
  const size_t off = ((size_t)bhk * Lk + r0) * D;
  const float s = quant_block<D, SAGE_K_BLOCK_ROWS, true>(k + off, k_i8 + off, rows,
                                                          k_mean + (size_t)bhk * D, red);
  if (threadIdx.x == 0) k_scale[blk] = s;
}

// ------------------------------------------------------------- launcher

size_t quant_workspace_bytes(int B, int Hkv, int Lk, int d) {
  const size_t nchunks = (size_t)(Lk + kMeanChunk - 1) / kMeanChunk;
  return (size_t)B * Hkv * nchunks * d * sizeof(long long);
}

template <int D>
static cudaError_t launch_quant_d(const QuantArgs& a, cudaStream_t st, int* launches) {
  const int BH = a.B * a.H, BHkv = a.B * a.Hkv;
  const int nchunks = (a.Lk + kMeanChunk - 1) / kMeanChunk;
  const int nqb = (a.Lq + SAGE_Q_BLOCK_ROWS - 1) / SAGE_Q_BLOCK_ROWS;
  const int nkb = (a.Lk + SAGE_K_BLOCK_ROWS - 1) / SAGE_K_BLOCK_ROWS;
  long long* part = static_cast<long long*>(a.workspace);
  const long long g1 = (long long)BHkv * nchunks + (long long)BH * nqb;
  const long long g3 = (long long)BHkv * nkb;
  if (g1 > 0x7fffffffLL || g3 > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  kmean_and_quant_q_kernel<D><<<(unsigned)g1, kQuantThreads, 0, st>>>(
      a.q, a.k, a.q_i8, a.q_scale, part, BHkv, BH, a.Lq, a.Lk, nchunks, nqb, a.c);
  kmean_finalize_kernel<D><<<BHkv, D, 0, st>>>(part, a.k_mean, a.Lk, nchunks);
  quant_k_kernel<D><<<(unsigned)g3, kQuantThreads, 0, st>>>(a.k, a.k_mean, a.k_i8, a.k_scale,
                                                           a.Lk, nkb);
  *launches += 3;
  return cudaGetLastError();
}

cudaError_t launch_quant(const QuantArgs& a, cudaStream_t st, int* launches) {
  return a.d == 128 ? launch_quant_d<128>(a, st, launches) : launch_quant_d<64>(a, st, launches);
}

}  // namespace sage
