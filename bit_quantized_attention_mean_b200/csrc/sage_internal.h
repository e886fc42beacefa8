// sage_internal.h -- launcher interfaces shared by the library's translation
// units (not part of the public ABI; see include/sage.h for that).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/sage.h"

#define SAGE_Q_BLOCK_ROWS 128
#define SAGE_K_BLOCK_ROWS 64

namespace sage {

// ------------------------------------------------ host-side argument checks

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape rules shared by every entry point: positive sizes, H a multiple of
// Hkv, d in {64, 128}, and element offsets / grid sizes that fit the
// kernels' index types.
inline sage_status check_shape(int B, int H, int Hkv, int Lq, int Lk, int d) {
  if (B < 1 || H < 1 || Hkv < 1 || Lq < 1 || Lk < 1) return SAGE_ERR_INVALID_ARG;
  if (H % Hkv != 0) return SAGE_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SAGE_ERR_UNSUPPORTED;
  const long long qn = (long long)B * H * Lq, kn = (long long)B * Hkv * Lk;
  if (qn * d > (1LL << 40) || kn * d > (1LL << 40)) return SAGE_ERR_INVALID_ARG;
  if (qn / 128 + 1 > 0x7fffffffLL || kn / 64 + 1 > 0x7fffffffLL) return SAGE_ERR_INVALID_ARG;
  return SAGE_OK;
}

// The quantization kernel's exact K column sums hold at most SAGE_MAX_LK keys
// per (batch, kv head); every call that quantizes K checks this first.
inline sage_status check_quant_len(int Lk) {
  return Lk > SAGE_MAX_LK ? SAGE_ERR_UNSUPPORTED : SAGE_OK;
}

// sm_100 device current (the library is built for sm_100a only).
inline sage_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SAGE_ERR_CUDA;
  if (major != 10 || minor != 0) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

// c = fl32(double(sm_scale) * log2(e)), folded into the Q scales.
inline float fold_constant(float sm_scale) {
  return (float)((double)sm_scale * 1.4426950408889634074);
}

// Records what sage_last_launch_count() reports for this thread.
void set_last_launch_count(int n);

struct QuantArgs {
  const __half* q;
  const __half* k;
  int8_t* q_i8;
  int8_t* k_i8;
  float* q_scale;
  float* k_scale;
  float* k_mean;
  int B, H, Hkv, Lq, Lk, d;
  float c;          // fl32(double(sm_scale) * log2(e)), folded into q_scale
  int q_block_rows; // rows per Q quantization block: 128, 64, 32 or 1
  // padded batches: rows / keys per batch entry ([B], <= Lq / Lk), or null
  const int* seqlens_q = nullptr;
  const int* seqlens_k = nullptr;
  // K only (smoothing + K blocks); the Q arguments are not used
  bool skip_q = false;
};

struct AttnArgs {
  const int8_t* q_i8;
  const int8_t* k_i8;
  const float* q_scale;
  const float* k_scale;
  const __half* v;
  __half* out;
  int B, H, Hkv, Lq, Lk, d;
  bool causal;
  int q_block_rows;   // rows per q_scale entry: 128, 64, 32 or 1
  bool pv_f16_accum;  // accumulate P V in fp16 (else fp32)
  bool pv_fp8 = false;            // P and V in E4M3 (v8t, v_scale below; v unused)
  const uint8_t* v8t = nullptr;   // E4M3 V^T [B, Hkv, d, 64 * ceil(Lk / 64)]
  const float* v_scale = nullptr; // [B, Hkv, d]
  // padded batches: rows / keys per batch entry ([B], <= Lq / Lk), or null
  const int* seqlens_q = nullptr;
  const int* seqlens_k = nullptr;
};

size_t quant_v_fp8_workspace_bytes(int B, int Hkv, int d);
// seqlens_k (device int32 [B], or null): per-entry key counts of a padded
// batch; maxima over each entry's own keys, codes past its count 0
cudaError_t launch_quant_v_fp8(const __half* v, uint8_t* v8t, float* v_scale, void* workspace,
                               int B, int Hkv, int Lk, int d, cudaStream_t st, int* launches,
                               const int* seqlens_k = nullptr);

inline bool valid_q_block_rows(int r) { return r == 128 || r == 64 || r == 32 || r == 1; }

// Few query tokens against a long key sequence: the query heads of a kv
// group packed into one tile (rows = (H / Hkv) * Lq <= 128), keys split over
// nsplit CTAs whose partial results a second kernel merges.
struct DecodeArgs {
  const int8_t* q_i8;
  const int8_t* k_i8;
  const float* q_scale;
  const float* k_scale;
  const __half* v;
  __half* out;
  float* o_part;    // [B*Hkv, nsplit, rows, d] partial outputs (nsplit > 1)
  float2* ml_part;  // [B*Hkv, nsplit, rows] running max (base 2) and sum
  int B, H, Hkv, Lq, Lk, d;
  bool causal;
  int q_block_rows;
  const int* seqlens = nullptr;  // [B] keys per batch entry (<= Lk), or null: all Lk
  // paged cache: k_i8/v are [num_pages, Hkv, 64, d], k_scale [num_pages, Hkv],
  // block_table [B, max_blocks] page indices, Lk = 64 * max_blocks
  const int* block_table = nullptr;
  int max_blocks = 0, num_pages = 0;
};

struct DecodePlan {
  int nsplit, split_tiles, rows;
  size_t o_bytes, ml_bytes;  // scratch for the partials (0 when nsplit = 1)
};

DecodePlan decode_plan(int B, int H, int Hkv, int Lq, int Lk, int d);
cudaError_t launch_decode(const DecodeArgs& a, const DecodePlan& p, cudaStream_t st,
                          int* launches);

// Each launcher adds the number of kernels it launched to *launches and
// returns the first CUDA error (cudaSuccess when every launch was accepted).
cudaError_t launch_quant(const QuantArgs& a, cudaStream_t st, int* launches);
cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st, int* launches);

// Launches a one-warp kernel whose bounded wait can never be satisfied and
// gives up after limit_ms (exercises the error path without a fault).
cudaError_t launch_wait_probe(int limit_ms, cudaStream_t st);

// Device status word written by kernels whose bounded waits gave up.
cudaError_t read_and_clear_device_status(int* value);
cudaError_t device_status_address(int** p);

}  // namespace sage
