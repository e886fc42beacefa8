// fp8.cu -- V to FP8 (E4M3) with one scale per channel, for the P V product
// with P and V in FP8 that the SageAttention2 description (the INT4 search
// results page, SageAttention2 entry) proposes.
//
// Per (batch, kv head) and channel c over all Lk tokens: a = max_t |V[t, c]|,
// r = fl32(448 / a), code = e4m3(fl32(V * r)) rounded to nearest even and
// saturated at 448, scale = fl32(a / 448) (a zero channel gives codes 0 and
// scale 0).  The codes are written channel-major, [B, Hkv, d, Lkp] with Lkp =
// 64 * ceil(Lk / 64) (padding code 0), so that a 64-key tile of one channel is
// one aligned 64-byte row: the K-major B operand of the tensor core's FP8 P V
// product.
//
// Two launches, HBM-bound: (1) channel maxima, each CTA reducing a range of
// tokens and merging into the global maxima with an integer atomicMax on the
// fp16 magnitude bits (exact and order-independent); (2) quantization and
// transposition of 64 x 64 tiles through shared memory.
//
// In a padded batch (per-entry key counts Lkb <= Lk) the maxima span the
// entry's own tokens only and every code past Lkb is 0, so V's padding is
// never read.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "sage_internal.h"

namespace sage {

constexpr int kAmaxTokens = 256;  // tokens per CTA of the maxima pass

// Largest |V| per channel, as fp16 magnitude bits, into amax[bh * d + c].
template <int D>
__global__ void __launch_bounds__(256)
v_amax_kernel(const __half* __restrict__ v, unsigned* __restrict__ amax, int Lk, int nchunk,
              const int* __restrict__ seqlens_k, int Hkv) {
  constexpr int TPR = D / 8;           // 16-byte vectors per token row
  constexpr int RPP = 256 / TPR;       // token rows per pass
  const int bh = blockIdx.x / nchunk, ch = blockIdx.x - bh * nchunk;
  const int Lkb = seqlens_k ? min(max(__ldg(seqlens_k + bh / Hkv), 0), Lk) : Lk;
  const int t0 = ch * kAmaxTokens, t1 = min(Lkb, t0 + kAmaxTokens);
  const int cg = threadIdx.x % TPR, rr = threadIdx.x / TPR;
  const uint4* base = reinterpret_cast<const uint4*>(v + (size_t)bh * Lk * D) + cg;
  uint32_t m[4] = {0u, 0u, 0u, 0u};  // two channels per word
  for (int t = t0 + rr; t < t1; t += RPP) {
    const uint4 raw = __ldcs(base + (size_t)t * TPR);
    m[0] = __vmaxu2(m[0], raw.x & 0x7fff7fffu);
    m[1] = __vmaxu2(m[1], raw.y & 0x7fff7fffu);
    m[2] = __vmaxu2(m[2], raw.z & 0x7fff7fffu);
    m[3] = __vmaxu2(m[3], raw.w & 0x7fff7fffu);
  }
  __shared__ uint32_t red[RPP][TPR][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) red[rr][cg][i] = m[i];
  __syncthreads();
  if (threadIdx.x < TPR * 4) {
    const int g = threadIdx.x / 4, i = threadIdx.x % 4;
    uint32_t w = 0u;
    for (int r = 0; r < RPP; ++r) w = __vmaxu2(w, red[r][g][i]);
    unsigned* dst = amax + (size_t)bh * D + g * 8 + 2 * i;
    atomicMax(dst, w & 0xffffu);
    atomicMax(dst + 1, w >> 16);
  }
}

// Quantizes a 64-token x 64-channel tile and writes it channel-major, each
// channel row padded to Lkp = 64 * ceil(Lk / 64) tokens (the padding holds
// code 0), so every 64-key tile of a channel is a whole, 64-byte aligned row.
template <int D>
__global__ void __launch_bounds__(256)
v_fp8_kernel(const __half* __restrict__ v, const unsigned* __restrict__ amax,
             uint8_t* __restrict__ v8t, float* __restrict__ v_scale, int Lk, int ntt,
             const int* __restrict__ seqlens_k, int Hkv) {
  constexpr int CT = D / 64;  // channel tiles per head
  const int tt = blockIdx.x % ntt, rest = blockIdx.x / ntt;
  const int ct = rest % CT, bh = rest / CT;
  const int t0 = tt * 64, c0 = ct * 64;
  const int Lkb = seqlens_k ? min(max(__ldg(seqlens_k + bh / Hkv), 0), Lk) : Lk;
  const int rows = min(64, Lkb - t0);  // <= 0: a tile of padding, all codes 0
  const size_t Lkp = (size_t)ntt * 64;
  __shared__ __half tile[64][64 + 8];  // [token][channel], padded rows
  __shared__ uint32_t codes[64][17];   // [channel][4-token word], padded rows
  __shared__ float rs[64];
  const int tid = threadIdx.x;
  if (tid < 64) {
    const unsigned ab = amax[(size_t)bh * D + c0 + tid];
    const float a = __fmul_rn(__uint_as_float(ab << 13), 0x1p112f);  // fp16 bits -> value
    rs[tid] = a > 0.f ? __fdiv_rn(448.f, a) : 0.f;
    if (tt == 0) v_scale[(size_t)bh * D + c0 + tid] = a > 0.f ? __fdiv_rn(a, 448.f) : 0.f;
  }
  // load: 64 tokens x 64 channels = 512 vectors of 8 channels (zeros past Lk)
  for (int idx = tid; idx < 64 * 8; idx += 256) {
    const int t = idx / 8, c8 = idx % 8;
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (t < rows)
      raw = __ldcs(reinterpret_cast<const uint4*>(v + ((size_t)bh * Lk + t0 + t) * D + c0) + c8);
    *reinterpret_cast<uint4*>(&tile[t][c8 * 8]) = raw;
  }
  __syncthreads();
  // codes: channel c, tokens [4q, 4q + 4) -> one word (token 4q in the low byte)
  for (int idx = tid; idx < 64 * 16; idx += 256) {
    const int c = idx % 64, q = idx / 64;
    const float r = rs[c];
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = __fmul_rn(__half2float(tile[4 * q + e][c]), r);
    uint16_t lo, hi;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(x[1]), "f"(x[0]));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(x[3]), "f"(x[2]));
    codes[c][q] = (uint32_t)lo | ((uint32_t)hi << 16);
  }
  __syncthreads();
  // store: 4 threads per channel row, 16 bytes each
  {
    const int c = tid / 4, part = tid % 4;
    uint4 w = make_uint4(codes[c][4 * part], codes[c][4 * part + 1], codes[c][4 * part + 2],
                         codes[c][4 * part + 3]);
    uint8_t* dst = v8t + ((size_t)bh * D + c0 + c) * Lkp + t0 + 16 * part;
    *reinterpret_cast<uint4*>(dst) = w;
  }
}

size_t quant_v_fp8_workspace_bytes(int B, int Hkv, int d) {
  return ((size_t)B * Hkv * d * sizeof(unsigned) + 255) & ~(size_t)255;
}

template <int D>
static cudaError_t launch_quant_v_fp8_d(const __half* v, uint8_t* v8t, float* v_scale,
                                        void* workspace, int B, int Hkv, int Lk,
                                        const int* seqlens_k, cudaStream_t st, int* launches) {
  unsigned* amax = static_cast<unsigned*>(workspace);
  cudaError_t e = cudaMemsetAsync(amax, 0, (size_t)B * Hkv * D * sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  const long long BH = (long long)B * Hkv;
  const int nchunk = (Lk + kAmaxTokens - 1) / kAmaxTokens;
  const int ntt = (Lk + 63) / 64;
  if (BH * nchunk > 0x7fffffffLL || BH * (D / 64) * ntt > 0x7fffffffLL)
    return cudaErrorInvalidConfiguration;
  v_amax_kernel<D><<<(unsigned)(BH * nchunk), 256, 0, st>>>(v, amax, Lk, nchunk, seqlens_k, Hkv);
  *launches += 1;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  v_fp8_kernel<D><<<(unsigned)(BH * (D / 64) * ntt), 256, 0, st>>>(v, amax, v8t, v_scale, Lk,
                                                                    ntt, seqlens_k, Hkv);
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_quant_v_fp8(const __half* v, uint8_t* v8t, float* v_scale, void* workspace,
                               int B, int Hkv, int Lk, int d, cudaStream_t st, int* launches,
                               const int* seqlens_k) {
  return d == 128 ? launch_quant_v_fp8_d<128>(v, v8t, v_scale, workspace, B, Hkv, Lk, seqlens_k,
                                              st, launches)
                  : launch_quant_v_fp8_d<64>(v, v8t, v_scale, workspace, B, Hkv, Lk, seqlens_k,
                                             st, launches);
}

}  // namespace sage
