// noalloc.cu -- sage_attn_fwd_noalloc: the whole forward pass without any
// device allocation at call time.
//
// sage_attn_fwd takes its scratch (int8 Q/K, block scales, K mean, K partial
// sums) from cudaMallocAsync on every call.  Some callers cannot allow that:
// a serving process that reserves its whole memory budget at start-up and
// treats any later allocation as an error (to keep latency and fragmentation
// predictable), or a plugin host that hands a library no allocator of its own.
// For them this entry point keeps the scratch in one fixed device array,
// g_noalloc_scratch, reserved when this file's module loads and held by every
// GPU that loads it until the process exits.
//
// Rules of use:
//   - The scratch holds kNoAllocScratchBytes (64 MiB).  Problems whose scratch
//     (sage_attn_workspace_size) exceeds it are rejected with
//     SAGE_ERR_INVALID_ARG before anything is launched.
//   - Every call shares the one array and leaves its contents behind.  Nothing
//     in it needs to start at zero: each call writes every byte it later reads.
//     Calls whose kernels overlap on the GPU (different streams without
//     ordering, or several host threads) race on the array and give wrong
//     results; order them on one stream.
//   - The first call on a device looks the array's device address up
//     (cudaGetSymbolAddress, once per device, with that device current).  Make
//     that first call before any stream capture begins.
//   - The caller still owns q, k, v and out; sage_last_launch_count does not
//     report this entry point.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/sage.h"
#include "sage_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 64ull << 20;

// Device-side scratch.  In host code this name is only a handle for
// cudaGetSymbolAddress, never a pointer to hand to a kernel.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once).
cudaError_t scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

size_t piece(size_t bytes) { return (bytes + 255) & ~(size_t)255; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" SAGE_API sage_status sage_attn_fwd_noalloc(const void* q, const void* k,
                                                      const void* v, void* out, int B, int H,
                                                      int Hkv, int Lq, int Lk, int d,
                                                      int causal, float sm_scale,
                                                      void* stream) {
  // --- arguments (host only; nothing touches the GPU before they pass)
  if (B < 1 || H < 1 || Hkv < 1 || Lq < 1 || Lk < 1 || H % Hkv != 0) return SAGE_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SAGE_ERR_UNSUPPORTED;
  if (!q || !k || !v || !out) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return SAGE_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;

  // --- scratch layout, each piece 256-byte aligned; reject what does not fit
  const size_t nqb = (size_t)(Lq + 127) / 128, nkb = (size_t)(Lk + 63) / 64;
  const size_t off_q = 0;
  const size_t off_k = off_q + piece((size_t)B * H * Lq * d);
  const size_t off_qs = off_k + piece((size_t)B * Hkv * Lk * d);
  const size_t off_ks = off_qs + piece((size_t)B * H * nqb * sizeof(float));
  const size_t off_m = off_ks + piece((size_t)B * Hkv * nkb * sizeof(float));
  const size_t off_p = off_m + piece((size_t)B * Hkv * d * sizeof(float));
  const size_t total = off_p + piece(sage::quant_workspace_bytes(B, Hkv, Lk, d));
  if (total > kNoAllocScratchBytes) return SAGE_ERR_INVALID_ARG;

  // --- device: sm_100 only, then the scratch address
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SAGE_ERR_CUDA;
  if (major != 10 || minor != 0) return SAGE_ERR_UNSUPPORTED;
  void* base = nullptr;
  if (scratch_on_current_device(&base) != cudaSuccess) return SAGE_ERR_CUDA;
  char* ws = static_cast<char*>(base);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int8_t* q_i8 = reinterpret_cast<int8_t*>(ws + off_q);
  int8_t* k_i8 = reinterpret_cast<int8_t*>(ws + off_k);
  float* q_scale = reinterpret_cast<float*>(ws + off_qs);
  float* k_scale = reinterpret_cast<float*>(ws + off_ks);
  float* k_mean = reinterpret_cast<float*>(ws + off_m);
  const float c = (float)((double)sm_scale * 1.4426950408889634074);  // sm_scale * log2(e)
  sage::QuantArgs qa{static_cast<const __half*>(q), static_cast<const __half*>(k), q_i8, k_i8,
                     q_scale, k_scale, k_mean, ws + off_p, B, H, Hkv, Lq, Lk, d, c,
                     SAGE_Q_BLOCK_ROWS};
  int launches = 0;
  cudaError_t e = sage::launch_quant(qa, s, &launches);
  if (e == cudaSuccess) {
    sage::AttnArgs aa{q_i8, k_i8, q_scale, k_scale, static_cast<const __half*>(v),
                      static_cast<__half*>(out), B, H, Hkv, Lq, Lk, d, causal == 1,
                      SAGE_Q_BLOCK_ROWS};
    e = sage::launch_attn(aa, s, &launches);
  }
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}
