// sage_api.cu -- the C ABI declared in include/sage.h: host-side argument
// validation, scratch management and dispatch to the sm_100a kernels.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/sage.h"
#include "sage_internal.h"

namespace {

thread_local int g_last_launches = 0;

using sage::aligned16;
using sage::check_device;
using sage::check_quant_len;
using sage::check_shape;
using sage::fold_constant;

size_t round_up(size_t x) { return (x + 255) & ~(size_t)255; }

// Accepted flag words of the _ex calls: 0, SAGE_PV_ACCUM_F16 or SAGE_PV_FP8.
bool valid_flags(unsigned f) { return f == 0u || f == SAGE_PV_ACCUM_F16 || f == SAGE_PV_FP8; }

size_t v8t_bytes(int B, int Hkv, int Lk, int d) {
  return (size_t)B * Hkv * d * (size_t)((Lk + 63) / 64 * 64);
}

constexpr int kMaxDevices = 64;
constexpr int kHostChunks = 8;  // chunks of (batch, kv head) groups in the host-buffer call

// Three non-blocking side streams per device for the host-buffer call (copy
// in, compute, copy out), created on first use and kept for the life of the
// process.
cudaStream_t* side_streams(int dev) {
  static cudaStream_t streams[kMaxDevices][3];
  static std::once_flag once[kMaxDevices];
  static bool ok[kMaxDevices];
  std::call_once(once[dev], [dev] {
    ok[dev] = true;
    for (int i = 0; i < 3; ++i)
      ok[dev] = ok[dev] &&
                cudaStreamCreateWithFlags(&streams[dev][i], cudaStreamNonBlocking) == cudaSuccess;
  });
  return ok[dev] ? streams[dev] : nullptr;
}

struct AttnWorkspace {
  size_t q_i8, k_i8, q_scale, k_scale, k_mean, total;
};

AttnWorkspace attn_workspace_layout(int B, int H, int Hkv, int Lq, int Lk, int d, int qbr) {
  AttnWorkspace w;
  const size_t nqb = (size_t)(Lq + qbr - 1) / qbr, nkb = (size_t)(Lk + 63) / 64;
  size_t off = 0;
  w.q_i8 = off;    off += round_up((size_t)B * H * Lq * d);
  w.k_i8 = off;    off += round_up((size_t)B * Hkv * Lk * d);
  w.q_scale = off; off += round_up((size_t)B * H * nqb * 4);
  w.k_scale = off; off += round_up((size_t)B * Hkv * nkb * 4);
  w.k_mean = off;  off += round_up((size_t)B * Hkv * d * 4);
  w.total = off;
  return w;
}

}  // namespace

namespace sage {
void set_last_launch_count(int n) { g_last_launches = n; }
}  // namespace sage

extern "C" {

const char* sage_status_string(sage_status s) {
  switch (s) {
    case SAGE_OK: return "SAGE_OK";
    case SAGE_ERR_INVALID_ARG: return "SAGE_ERR_INVALID_ARG";
    case SAGE_ERR_UNSUPPORTED: return "SAGE_ERR_UNSUPPORTED";
    case SAGE_ERR_CUDA: return "SAGE_ERR_CUDA";
    case SAGE_ERR_TIMEOUT: return "SAGE_ERR_TIMEOUT";
  }
  return "SAGE_ERR_UNKNOWN";
}

int sage_last_launch_count(void) { return g_last_launches; }

size_t sage_workspace_size(int B, int H, int Hkv, int Lq, int Lk, int d) {
  if (check_shape(B, H, Hkv, Lq, Lk, d) != SAGE_OK) return 0;
  return attn_workspace_layout(B, H, Hkv, Lq, Lk, d, SAGE_Q_BLOCK).total;
}

sage_status sage_quant_qk(const void* q, const void* k, int8_t* q_i8, int8_t* k_i8, float* q_scale,
                          float* k_scale, float* k_mean, int B, int H, int Hkv, int Lq, int Lk,
                          int d, float sm_scale, void* stream) {
  return sage_quant_qk_qblock(q, k, q_i8, k_i8, q_scale, k_scale, k_mean, B, H, Hkv, Lq, Lk, d,
                              sm_scale, SAGE_Q_BLOCK, stream);
}

sage_status sage_quant_qk_qblock(const void* q, const void* k, int8_t* q_i8, int8_t* k_i8,
                                 float* q_scale, float* k_scale, float* k_mean, int B, int H,
                                 int Hkv, int Lq, int Lk, int d, float sm_scale, int q_block_rows,
                                 void* stream) {
  return sage_quant_qk_varlen(q, k, q_i8, k_i8, q_scale, k_scale, k_mean, nullptr, nullptr, B, H,
                              Hkv, Lq, Lk, d, sm_scale, q_block_rows, stream);
}

sage_status sage_quant_qk_varlen(const void* q, const void* k, int8_t* q_i8, int8_t* k_i8,
                                 float* q_scale, float* k_scale, float* k_mean,
                                 const int* seqlens_q, const int* seqlens_k, int B, int H,
                                 int Hkv, int Lq, int Lk, int d, float sm_scale, int q_block_rows,
                                 void* stream) {
  g_last_launches = 0;
  sage_status st = check_shape(B, H, Hkv, Lq, Lk, d);
  if (st != SAGE_OK) return st;
  if ((st = check_quant_len(Lk)) != SAGE_OK) return st;
  if (!sage::valid_q_block_rows(q_block_rows)) return SAGE_ERR_INVALID_ARG;
  if (!q || !k || !q_i8 || !k_i8 || !q_scale || !k_scale || !k_mean) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_i8) || !aligned16(k_i8) ||
      !aligned16(q_scale) || !aligned16(k_scale) || !aligned16(k_mean))
    return SAGE_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  if ((st = check_device()) != SAGE_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  sage::QuantArgs a{static_cast<const __half*>(q), static_cast<const __half*>(k), q_i8, k_i8,
                    q_scale, k_scale, k_mean, B, H, Hkv, Lq, Lk, d, fold_constant(sm_scale),
                    q_block_rows, seqlens_q, seqlens_k};
  int launches = 0;
  cudaError_t e = sage::launch_quant(a, s, &launches);
  g_last_launches = launches;
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

sage_status sage_attn_fwd_prequant(const int8_t* q_i8, const int8_t* k_i8, const float* q_scale,
                                   const float* k_scale, const void* v, void* out, int B, int H,
                                   int Hkv, int Lq, int Lk, int d, int causal, void* stream) {
  return sage_attn_fwd_prequant_qblock(q_i8, k_i8, q_scale, k_scale, v, out, B, H, Hkv, Lq, Lk, d,
                                       causal, SAGE_Q_BLOCK, stream);
}

sage_status sage_attn_fwd_prequant_qblock(const int8_t* q_i8, const int8_t* k_i8,
                                          const float* q_scale, const float* k_scale,
                                          const void* v, void* out, int B, int H, int Hkv, int Lq,
                                          int Lk, int d, int causal, int q_block_rows,
                                          void* stream) {
  return sage_attn_fwd_prequant_ex(q_i8, k_i8, q_scale, k_scale, v, out, B, H, Hkv, Lq, Lk, d,
                                   causal, q_block_rows, 0u, stream);
}

sage_status sage_attn_fwd_prequant_ex(const int8_t* q_i8, const int8_t* k_i8,
                                      const float* q_scale, const float* k_scale, const void* v,
                                      void* out, int B, int H, int Hkv, int Lq, int Lk, int d,
                                      int causal, int q_block_rows, unsigned flags, void* stream) {
  return sage_attn_fwd_prequant_varlen(q_i8, k_i8, q_scale, k_scale, v, out, nullptr, nullptr, B,
                                       H, Hkv, Lq, Lk, d, causal, q_block_rows, flags, stream);
}

sage_status sage_attn_fwd_prequant_varlen(const int8_t* q_i8, const int8_t* k_i8,
                                          const float* q_scale, const float* k_scale,
                                          const void* v, void* out, const int* seqlens_q,
                                          const int* seqlens_k, int B, int H, int Hkv, int Lq,
                                          int Lk, int d, int causal, int q_block_rows,
                                          unsigned flags, void* stream) {
  g_last_launches = 0;
  sage_status st = check_shape(B, H, Hkv, Lq, Lk, d);
  if (st != SAGE_OK) return st;
  if (!sage::valid_q_block_rows(q_block_rows)) return SAGE_ERR_INVALID_ARG;
  if (!valid_flags(flags) || flags == SAGE_PV_FP8) return SAGE_ERR_INVALID_ARG;
  if (!q_i8 || !k_i8 || !q_scale || !k_scale || !v || !out) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q_i8) || !aligned16(k_i8) || !aligned16(v) || !aligned16(out) ||
      !aligned16(q_scale) || !aligned16(k_scale))
    return SAGE_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if ((st = check_device()) != SAGE_OK) return st;
  sage::AttnArgs a{q_i8, k_i8, q_scale, k_scale, static_cast<const __half*>(v),
                   static_cast<__half*>(out), B, H, Hkv, Lq, Lk, d, causal == 1, q_block_rows,
                   (flags & SAGE_PV_ACCUM_F16) != 0u};
  a.seqlens_q = seqlens_q;
  a.seqlens_k = seqlens_k;
  int launches = 0;
  cudaError_t e = sage::launch_attn(a, static_cast<cudaStream_t>(stream), &launches);
  g_last_launches = launches;
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

sage_status sage_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int H,
                          int Hkv, int Lq, int Lk, int d, int causal, float sm_scale,
                          void* stream) {
  return sage_attn_fwd_qblock(q, k, v, out, B, H, Hkv, Lq, Lk, d, causal, sm_scale, SAGE_Q_BLOCK,
                              stream);
}

sage_status sage_attn_fwd_qblock(const void* q, const void* k, const void* v, void* out, int B,
                                 int H, int Hkv, int Lq, int Lk, int d, int causal, float sm_scale,
                                 int q_block_rows, void* stream) {
  return sage_attn_fwd_ex(q, k, v, out, B, H, Hkv, Lq, Lk, d, causal, sm_scale, q_block_rows, 0u,
                          stream);
}

sage_status sage_attn_fwd_ex(const void* q, const void* k, const void* v, void* out, int B, int H,
                             int Hkv, int Lq, int Lk, int d, int causal, float sm_scale,
                             int q_block_rows, unsigned flags, void* stream) {
  return sage_attn_fwd_varlen(q, k, v, out, nullptr, nullptr, B, H, Hkv, Lq, Lk, d, causal,
                              sm_scale, q_block_rows, flags, stream);
}

sage_status sage_attn_fwd_varlen(const void* q, const void* k, const void* v, void* out,
                                 const int* seqlens_q, const int* seqlens_k, int B, int H,
                                 int Hkv, int Lq, int Lk, int d, int causal, float sm_scale,
                                 int q_block_rows, unsigned flags, void* stream) {
  g_last_launches = 0;
  sage_status st = check_shape(B, H, Hkv, Lq, Lk, d);
  if (st != SAGE_OK) return st;
  if ((st = check_quant_len(Lk)) != SAGE_OK) return st;
  if (!sage::valid_q_block_rows(q_block_rows)) return SAGE_ERR_INVALID_ARG;
  if (!valid_flags(flags)) return SAGE_ERR_INVALID_ARG;
  if (!q || !k || !v || !out) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return SAGE_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  if ((st = check_device()) != SAGE_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const AttnWorkspace w = attn_workspace_layout(B, H, Hkv, Lq, Lk, d, q_block_rows);
  const bool fp8 = flags == SAGE_PV_FP8;
  // E4M3 V^T, its channel scales and the maxima scratch after the common part
  const size_t v8_off = w.total, vs_off = v8_off + round_up(v8t_bytes(B, Hkv, Lk, d));
  const size_t vm_off = vs_off + round_up((size_t)B * Hkv * d * 4);
  const size_t total = fp8 ? vm_off + sage::quant_v_fp8_workspace_bytes(B, Hkv, d) : w.total;
  char* ws = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void**>(&ws), total, s) != cudaSuccess)
    return SAGE_ERR_CUDA;
  int8_t* q_i8 = reinterpret_cast<int8_t*>(ws + w.q_i8);
  int8_t* k_i8 = reinterpret_cast<int8_t*>(ws + w.k_i8);
  float* q_scale = reinterpret_cast<float*>(ws + w.q_scale);
  float* k_scale = reinterpret_cast<float*>(ws + w.k_scale);
  float* k_mean = reinterpret_cast<float*>(ws + w.k_mean);
  sage::QuantArgs qa{static_cast<const __half*>(q), static_cast<const __half*>(k), q_i8, k_i8,
                     q_scale, k_scale, k_mean, B, H, Hkv, Lq, Lk, d,
                     fold_constant(sm_scale), q_block_rows, seqlens_q, seqlens_k};
  int launches = 0;
  cudaError_t e = sage::launch_quant(qa, s, &launches);
  uint8_t* v8t = reinterpret_cast<uint8_t*>(ws + v8_off);
  float* v_scale = reinterpret_cast<float*>(ws + vs_off);
  if (e == cudaSuccess && fp8)
    e = sage::launch_quant_v_fp8(static_cast<const __half*>(v), v8t, v_scale, ws + vm_off, B, Hkv,
                                 Lk, d, s, &launches, seqlens_k);
  if (e == cudaSuccess) {
    sage::AttnArgs aa{q_i8, k_i8, q_scale, k_scale, static_cast<const __half*>(v),
                      static_cast<__half*>(out), B, H, Hkv, Lq, Lk, d, causal == 1,
                      q_block_rows, flags == SAGE_PV_ACCUM_F16};
    aa.seqlens_q = seqlens_q;
    aa.seqlens_k = seqlens_k;
    if (fp8) {
      aa.pv_fp8 = true;
      aa.v8t = v8t;
      aa.v_scale = v_scale;
    }
    e = sage::launch_attn(aa, s, &launches);
  }
  if (cudaFreeAsync(ws, s) != cudaSuccess && e == cudaSuccess) e = cudaErrorUnknown;
  g_last_launches = launches;
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

sage_status sage_quant_k(const void* k, int8_t* k_i8, float* k_scale, float* k_mean, int B,
                         int Hkv, int Lk, int d, void* stream) {
  g_last_launches = 0;
  sage_status st = check_shape(B, Hkv, Hkv, 1, Lk, d);
  if (st != SAGE_OK) return st;
  if ((st = check_quant_len(Lk)) != SAGE_OK) return st;
  if (!k || !k_i8 || !k_scale || !k_mean) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(k_i8) || !aligned16(k_scale) || !aligned16(k_mean))
    return SAGE_ERR_INVALID_ARG;
  if ((st = check_device()) != SAGE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  sage::QuantArgs a{nullptr, static_cast<const __half*>(k), nullptr, k_i8, nullptr, k_scale,
                    k_mean, B, Hkv, Hkv, 1, Lk, d, 1.f, SAGE_Q_BLOCK};
  a.skip_q = true;
  int launches = 0;
  cudaError_t e = sage::launch_quant(a, s, &launches);
  g_last_launches = launches;
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

size_t sage_attn_decode_workspace_size(int B, int H, int Hkv, int Lq, int Lk, int d) {
  if (check_shape(B, H, Hkv, Lq, Lk, d) != SAGE_OK || (long long)(H / Hkv) * Lq > 128) return 0;
  const sage::DecodePlan p = sage::decode_plan(B, H, Hkv, Lq, Lk, d);
  return p.o_bytes + p.ml_bytes;
}

sage_status sage_attn_decode_prequant(const int8_t* q_i8, const int8_t* k_i8,
                                      const float* q_scale, const float* k_scale, const void* v,
                                      void* out, int B, int H, int Hkv, int Lq, int Lk, int d,
                                      int causal, int q_block_rows, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  return sage_attn_decode_prequant_varlen(q_i8, k_i8, q_scale, k_scale, v, out, nullptr, B, H,
                                          Hkv, Lq, Lk, d, causal, q_block_rows, workspace,
                                          workspace_bytes, stream);
}

sage_status sage_attn_decode_prequant_varlen(const int8_t* q_i8, const int8_t* k_i8,
                                             const float* q_scale, const float* k_scale,
                                             const void* v, void* out, const int* seqlens_k,
                                             int B, int H, int Hkv, int Lq, int Lk, int d,
                                             int causal, int q_block_rows, void* workspace,
                                             size_t workspace_bytes, void* stream) {
  g_last_launches = 0;
  sage_status st = check_shape(B, H, Hkv, Lq, Lk, d);
  if (st != SAGE_OK) return st;
  if ((long long)(H / Hkv) * Lq > 128) return SAGE_ERR_UNSUPPORTED;
  if (!sage::valid_q_block_rows(q_block_rows)) return SAGE_ERR_INVALID_ARG;
  if (!q_i8 || !k_i8 || !q_scale || !k_scale || !v || !out) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q_i8) || !aligned16(k_i8) || !aligned16(v) || !aligned16(out) ||
      !aligned16(q_scale) || !aligned16(k_scale))
    return SAGE_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if ((st = check_device()) != SAGE_OK) return st;
  const sage::DecodePlan p = sage::decode_plan(B, H, Hkv, Lq, Lk, d);
  const size_t need = p.o_bytes + p.ml_bytes;
  if (workspace && (workspace_bytes < need || !aligned16(workspace))) return SAGE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const bool own = !ws && need > 0;
  if (own && cudaMallocAsync(reinterpret_cast<void**>(&ws), need, s) != cudaSuccess)
    return SAGE_ERR_CUDA;
  sage::DecodeArgs a{q_i8, k_i8, q_scale, k_scale, static_cast<const __half*>(v),
                     static_cast<__half*>(out), need ? reinterpret_cast<float*>(ws) : nullptr,
                     need ? reinterpret_cast<float2*>(ws + p.o_bytes) : nullptr,
                     B, H, Hkv, Lq, Lk, d, causal == 1, q_block_rows, seqlens_k};
  int launches = 0;
  cudaError_t e = sage::launch_decode(a, p, s, &launches);
  if (own && cudaFreeAsync(ws, s) != cudaSuccess && e == cudaSuccess) e = cudaErrorUnknown;
  g_last_launches = launches;
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

sage_status sage_attn_decode_prequant_paged(const int8_t* q_i8, const float* q_scale,
                                            const int8_t* k_pages, const float* k_scale_pages,
                                            const void* v_pages, const int* block_table,
                                            const int* seqlens_k, void* out, int B, int H,
                                            int Hkv, int Lq, int num_pages, int max_blocks, int d,
                                            int causal, int q_block_rows, void* workspace,
                                            size_t workspace_bytes, void* stream) {
  g_last_launches = 0;
  if (num_pages < 1 || max_blocks < 1 || (long long)max_blocks * 64 > 0x7fffffffLL)
    return SAGE_ERR_INVALID_ARG;
  const int Lk = max_blocks * 64;
  sage_status st = check_shape(B, H, Hkv, Lq, Lk, d);
  if (st != SAGE_OK) return st;
  if ((long long)num_pages * Hkv * 64 * d > (1LL << 40)) return SAGE_ERR_INVALID_ARG;
  if ((long long)(H / Hkv) * Lq > 128) return SAGE_ERR_UNSUPPORTED;
  if (!sage::valid_q_block_rows(q_block_rows)) return SAGE_ERR_INVALID_ARG;
  if (!q_i8 || !q_scale || !k_pages || !k_scale_pages || !v_pages || !block_table || !seqlens_k ||
      !out)
    return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q_i8) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(out) ||
      !aligned16(q_scale) || !aligned16(k_scale_pages))
    return SAGE_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if ((st = check_device()) != SAGE_OK) return st;
  const sage::DecodePlan p = sage::decode_plan(B, H, Hkv, Lq, Lk, d);
  const size_t need = p.o_bytes + p.ml_bytes;
  if (workspace && (workspace_bytes < need || !aligned16(workspace))) return SAGE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const bool own = !ws && need > 0;
  if (own && cudaMallocAsync(reinterpret_cast<void**>(&ws), need, s) != cudaSuccess)
    return SAGE_ERR_CUDA;
  sage::DecodeArgs a{q_i8, k_pages, q_scale, k_scale_pages, static_cast<const __half*>(v_pages),
                     static_cast<__half*>(out), need ? reinterpret_cast<float*>(ws) : nullptr,
                     need ? reinterpret_cast<float2*>(ws + p.o_bytes) : nullptr,
                     B, H, Hkv, Lq, Lk, d, causal == 1, q_block_rows, seqlens_k};
  a.block_table = block_table;
  a.max_blocks = max_blocks;
  a.num_pages = num_pages;
  int launches = 0;
  cudaError_t e = sage::launch_decode(a, p, s, &launches);
  if (own && cudaFreeAsync(ws, s) != cudaSuccess && e == cudaSuccess) e = cudaErrorUnknown;
  g_last_launches = launches;
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

sage_status sage_attn_decode(const void* q, const void* k, const void* v, void* out, int B, int H,
                             int Hkv, int Lq, int Lk, int d, int causal, float sm_scale,
                             int q_block_rows, void* stream) {
  g_last_launches = 0;
  sage_status st = check_shape(B, H, Hkv, Lq, Lk, d);
  if (st != SAGE_OK) return st;
  if ((st = check_quant_len(Lk)) != SAGE_OK) return st;
  if ((long long)(H / Hkv) * Lq > 128) return SAGE_ERR_UNSUPPORTED;
  if (!sage::valid_q_block_rows(q_block_rows)) return SAGE_ERR_INVALID_ARG;
  if (!q || !k || !v || !out) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return SAGE_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  if ((st = check_device()) != SAGE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const AttnWorkspace w = attn_workspace_layout(B, H, Hkv, Lq, Lk, d, q_block_rows);
  const sage::DecodePlan p = sage::decode_plan(B, H, Hkv, Lq, Lk, d);
  const size_t dec = p.o_bytes + p.ml_bytes;
  char* ws = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void**>(&ws), w.total + dec, s) != cudaSuccess)
    return SAGE_ERR_CUDA;
  int8_t* q_i8 = reinterpret_cast<int8_t*>(ws + w.q_i8);
  int8_t* k_i8 = reinterpret_cast<int8_t*>(ws + w.k_i8);
  float* q_scale = reinterpret_cast<float*>(ws + w.q_scale);
  float* k_scale = reinterpret_cast<float*>(ws + w.k_scale);
  float* k_mean = reinterpret_cast<float*>(ws + w.k_mean);
  sage::QuantArgs qa{static_cast<const __half*>(q), static_cast<const __half*>(k), q_i8, k_i8,
                     q_scale, k_scale, k_mean, B, H, Hkv, Lq, Lk, d,
                     fold_constant(sm_scale), q_block_rows};
  int launches = 0;
  cudaError_t e = sage::launch_quant(qa, s, &launches);
  if (e == cudaSuccess) {
    char* dws = ws + w.total;
    sage::DecodeArgs da{q_i8, k_i8, q_scale, k_scale, static_cast<const __half*>(v),
                        static_cast<__half*>(out), dec ? reinterpret_cast<float*>(dws) : nullptr,
                        dec ? reinterpret_cast<float2*>(dws + p.o_bytes) : nullptr,
                        B, H, Hkv, Lq, Lk, d, causal == 1, q_block_rows};
    e = sage::launch_decode(da, p, s, &launches);
  }
  if (cudaFreeAsync(ws, s) != cudaSuccess && e == cudaSuccess) e = cudaErrorUnknown;
  g_last_launches = launches;
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

size_t sage_quant_v_fp8_workspace_size(int B, int Hkv, int d) {
  if (B < 1 || Hkv < 1 || (d != 64 && d != 128)) return 0;
  return sage::quant_v_fp8_workspace_bytes(B, Hkv, d);
}

sage_status sage_quant_v_fp8(const void* v, uint8_t* v8t, float* v_scale, int B, int Hkv, int Lk,
                             int d, void* workspace, size_t workspace_bytes, void* stream) {
  g_last_launches = 0;
  sage_status st = check_shape(B, Hkv, Hkv, 1, Lk, d);
  if (st != SAGE_OK) return st;
  if (!v || !v8t || !v_scale) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(v) || !aligned16(v8t) || !aligned16(v_scale)) return SAGE_ERR_INVALID_ARG;
  const size_t need = sage::quant_v_fp8_workspace_bytes(B, Hkv, d);
  if (workspace && (workspace_bytes < need || !aligned16(workspace))) return SAGE_ERR_INVALID_ARG;
  if ((st = check_device()) != SAGE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = workspace;
  const bool own = !ws;
  if (own && cudaMallocAsync(&ws, need, s) != cudaSuccess) return SAGE_ERR_CUDA;
  int launches = 0;
  cudaError_t e = sage::launch_quant_v_fp8(static_cast<const __half*>(v), v8t, v_scale, ws, B,
                                           Hkv, Lk, d, s, &launches);
  if (own && cudaFreeAsync(ws, s) != cudaSuccess && e == cudaSuccess) e = cudaErrorUnknown;
  g_last_launches = launches;
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

sage_status sage_attn_fwd_prequant_fp8pv(const int8_t* q_i8, const int8_t* k_i8,
                                         const float* q_scale, const float* k_scale,
                                         const uint8_t* v8t, const float* v_scale, void* out,
                                         int B, int H, int Hkv, int Lq, int Lk, int d, int causal,
                                         int q_block_rows, void* stream) {
  g_last_launches = 0;
  sage_status st = check_shape(B, H, Hkv, Lq, Lk, d);
  if (st != SAGE_OK) return st;
  if (!sage::valid_q_block_rows(q_block_rows)) return SAGE_ERR_INVALID_ARG;
  if (!q_i8 || !k_i8 || !q_scale || !k_scale || !v8t || !v_scale || !out)
    return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q_i8) || !aligned16(k_i8) || !aligned16(v8t) || !aligned16(out) ||
      !aligned16(q_scale) || !aligned16(k_scale) || !aligned16(v_scale))
    return SAGE_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if ((st = check_device()) != SAGE_OK) return st;
  sage::AttnArgs a{q_i8, k_i8, q_scale, k_scale, nullptr, static_cast<__half*>(out), B, H, Hkv,
                   Lq, Lk, d, causal == 1, q_block_rows, false};
  a.pv_fp8 = true;
  a.v8t = v8t;
  a.v_scale = v_scale;
  int launches = 0;
  cudaError_t e = sage::launch_attn(a, static_cast<cudaStream_t>(stream), &launches);
  g_last_launches = launches;
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

sage_status sage_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                               void* out_host, int B, int H, int Hkv, int Lq, int Lk, int d,
                               int causal, float sm_scale, void* stream) {
  return sage_attn_fwd_host_qblock(q_host, k_host, v_host, out_host, B, H, Hkv, Lq, Lk, d, causal,
                                   sm_scale, SAGE_Q_BLOCK, stream);
}

sage_status sage_attn_fwd_host_qblock(const void* q_host, const void* k_host,
                                      const void* v_host, void* out_host, int B, int H, int Hkv,
                                      int Lq, int Lk, int d, int causal, float sm_scale,
                                      int q_block_rows, void* stream) {
  g_last_launches = 0;
  sage_status st = check_shape(B, H, Hkv, Lq, Lk, d);
  if (st != SAGE_OK) return st;
  if ((st = check_quant_len(Lk)) != SAGE_OK) return st;
  if (!sage::valid_q_block_rows(q_block_rows)) return SAGE_ERR_INVALID_ARG;
  if (!q_host || !k_host || !v_host || !out_host) return SAGE_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  if ((st = check_device()) != SAGE_OK) return st;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SAGE_ERR_CUDA;
  cudaStream_t* side = side_streams(dev);
  if (!side) return SAGE_ERR_CUDA;

  // Every (batch, kv head) group is independent: its K mean, its blocks and
  // its query heads.  Groups are processed in chunks through a three-stage
  // pipeline on side streams: copy-in (all host->device copies back to back),
  // compute (quantization + attention of chunk i once its copies are in) and
  // copy-out (chunk i's output once computed), so the copy engines stay busy
  // while the kernels run.  Query heads of groups [g0, g1) are the flat heads
  // [g0 G, g1 G) and kv heads are [g0, g1), both contiguous, so a chunk is the
  // problem B = 1, H = (g1 - g0) G, Hkv = g1 - g0.
  const int G = H / Hkv;
  const int groups = B * Hkv;
  const int nchunk = groups < kHostChunks ? groups : kHostChunks;
  const int per = (groups + nchunk - 1) / nchunk;
  const size_t qh = (size_t)Lq * d * 2, kh = (size_t)Lk * d * 2;  // bytes per head
  const size_t qb = (size_t)B * H * qh, kb = (size_t)B * Hkv * kh;
  const AttnWorkspace w = attn_workspace_layout(1, per * G, per, Lq, Lk, d, q_block_rows);
  const size_t total = round_up(qb) * 2 + round_up(kb) * 2 + w.total;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* buf = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void**>(&buf), total, s) != cudaSuccess) return SAGE_ERR_CUDA;
  char* dq = buf;
  char* dout = dq + round_up(qb);
  char* dk = dout + round_up(qb);
  char* dv = dk + round_up(kb);
  char* ws = dv + round_up(kb);
  // events: [0, nchunk) copies in, [nchunk, 2 nchunk) computed, then start
  // and the three stage ends
  const int nev = 2 * nchunk + 4;
  cudaEvent_t ev[2 * kHostChunks + 4];
  int made = 0;
  cudaError_t e = cudaSuccess;
  for (; made < nev && e == cudaSuccess; ++made)
    e = cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming);
  if (e != cudaSuccess) {
    for (int j = 0; j < made - 1; ++j) cudaEventDestroy(ev[j]);
    cudaFreeAsync(buf, s);
    return SAGE_ERR_CUDA;
  }
  cudaEvent_t* ev_in = ev;
  cudaEvent_t* ev_done = ev + nchunk;
  cudaEvent_t ev_start = ev[2 * nchunk];
  e = cudaEventRecord(ev_start, s);  // the buffer exists on `stream` from here
  for (int i = 0; i < 3 && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(side[i], ev_start, 0);
  cudaStream_t cin = side[0], comp = side[1], cout = side[2];
  const float c = fold_constant(sm_scale);
  int launches = 0;
  for (int ci = 0; ci < nchunk && e == cudaSuccess; ++ci) {
    const int g0 = ci * per, g1 = g0 + per < groups ? g0 + per : groups;
    const int n = g1 > g0 ? g1 - g0 : 0;
    const size_t qo = (size_t)g0 * G * qh, ko = (size_t)g0 * kh;
    if (n > 0) {
      e = cudaMemcpyAsync(dk + ko, static_cast<const char*>(k_host) + ko, n * kh,
                          cudaMemcpyHostToDevice, cin);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(dq + qo, static_cast<const char*>(q_host) + qo, n * G * qh,
                            cudaMemcpyHostToDevice, cin);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(dv + ko, static_cast<const char*>(v_host) + ko, n * kh,
                            cudaMemcpyHostToDevice, cin);
    }
    if (e == cudaSuccess) e = cudaEventRecord(ev_in[ci], cin);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(comp, ev_in[ci], 0);
    if (e == cudaSuccess && n > 0) {
      int8_t* q_i8 = reinterpret_cast<int8_t*>(ws + w.q_i8);
      int8_t* k_i8 = reinterpret_cast<int8_t*>(ws + w.k_i8);
      float* q_scale = reinterpret_cast<float*>(ws + w.q_scale);
      float* k_scale = reinterpret_cast<float*>(ws + w.k_scale);
      float* k_mean = reinterpret_cast<float*>(ws + w.k_mean);
      sage::QuantArgs qa{reinterpret_cast<const __half*>(dq + qo),
                         reinterpret_cast<const __half*>(dk + ko), q_i8, k_i8, q_scale, k_scale,
                         k_mean, 1, n * G, n, Lq, Lk, d, c, q_block_rows};
      e = sage::launch_quant(qa, comp, &launches);
      if (e == cudaSuccess) {
        sage::AttnArgs aa{q_i8, k_i8, q_scale, k_scale, reinterpret_cast<const __half*>(dv + ko),
                          reinterpret_cast<__half*>(dout + qo), 1, n * G, n, Lq, Lk, d,
                          causal == 1, q_block_rows, false};
        e = sage::launch_attn(aa, comp, &launches);
      }
    }
    if (e == cudaSuccess) e = cudaEventRecord(ev_done[ci], comp);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cout, ev_done[ci], 0);
    if (e == cudaSuccess && n > 0)
      e = cudaMemcpyAsync(static_cast<char*>(out_host) + qo, dout + qo, n * G * qh,
                          cudaMemcpyDeviceToHost, cout);
  }
  // `stream` resumes after the three stages; then the buffer is released
  for (int i = 0; i < 3; ++i) {
    cudaEvent_t end = ev[2 * nchunk + 1 + i];
    if (cudaEventRecord(end, side[i]) != cudaSuccess || cudaStreamWaitEvent(s, end, 0) != cudaSuccess)
      if (e == cudaSuccess) e = cudaErrorUnknown;
  }
  if (cudaFreeAsync(buf, s) != cudaSuccess && e == cudaSuccess) e = cudaErrorUnknown;
  for (int i = 0; i < nev; ++i) cudaEventDestroy(ev[i]);
  g_last_launches = launches;
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

sage_status sage_debug_wait_timeout(int limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 2000) return SAGE_ERR_INVALID_ARG;
  sage_status st = check_device();
  if (st != SAGE_OK) return st;
  return sage::launch_wait_probe(limit_ms, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SAGE_OK
             : SAGE_ERR_CUDA;
}

sage_status sage_check_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SAGE_ERR_CUDA;
  int v = 0;
  if (sage::read_and_clear_device_status(&v) != cudaSuccess) return SAGE_ERR_CUDA;
  return v != 0 ? SAGE_ERR_TIMEOUT : SAGE_OK;
}

}  // extern "C"
