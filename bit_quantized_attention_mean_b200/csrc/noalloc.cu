// noalloc.cu -- sage_attn_fwd_noalloc: the whole forward pass without any
// device allocation at call time.
//
// sage_attn_fwd takes its scratch (int8 Q/K, block scales, K mean) from
// cudaMallocAsync on every call.  Some callers cannot allow that:
// a serving process that reserves its whole memory budget at start-up and
// treats any later allocation as an error (to keep latency and fragmentation
// predictable), or a plugin host that hands a library no allocator of its own.
// For them this entry point keeps the scratch in one fixed device array,
// g_noalloc_scratch, reserved when this file's module loads and held by every
// GPU that loads it until the process exits.
//
// Rules of use:
//   - The scratch holds kNoAllocScratchBytes (64 MiB).  Problems whose scratch
//     (sage_workspace_size) exceeds it are rejected with
//     SAGE_ERR_INVALID_ARG before anything is launched; so are the shapes,
//     pointers and scalars every other entry point rejects.
//   - Every call shares the one array and leaves its contents behind.  Nothing
//     in it needs to start at zero: each call writes every byte it later reads.
//     Calls whose kernels overlap on the GPU (different streams without
//     ordering, or several host threads) race on the array and give wrong
//     results; order them on one stream.
//   - The first call on a device (and the first after that device's context
//     was destroyed and created again, e.g. by cudaDeviceReset) looks the
//     array's device address up with cudaGetSymbolAddress, with that device
//     current.  Make that first call before any stream capture begins.
//   - The caller still owns q, k, v and out; sage_last_launch_count reports
//     the kernels a successful call launched, as for the other calls.
#include <cuda.h>
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

// The address is cached per device together with the unique id of the
// context it was looked up in: a module reloaded into a new context may place
// the array elsewhere.
struct ScratchSlot {
  unsigned long long ctx_id = 0;
  void* ptr = nullptr;
};
std::mutex g_scratch_mu;
ScratchSlot g_scratch[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<Fn>(p);
  return nullptr;
}

// Unique id of the calling thread's current context; false when none is
// current (the runtime has not bound its primary context yet).
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_noalloc_scratch in the current device's current
// context.  cudaGetSymbolAddress, the only runtime call made here besides
// cudaGetDevice, also binds the primary context when none is current yet.
cudaError_t scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch[dev];
  unsigned long long id = 0;
  const bool have_ctx = current_context_id(&id);
  if (!have_ctx || slot.ptr == nullptr || slot.ctx_id != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (!current_context_id(&id)) return cudaErrorDeviceUninitialized;
    slot.ctx_id = id;
    slot.ptr = p;
  }
  *out = slot.ptr;
  return cudaSuccess;
}

size_t piece(size_t bytes) { return (bytes + 255) & ~(size_t)255; }

}  // namespace

extern "C" SAGE_API sage_status sage_attn_fwd_noalloc(const void* q, const void* k,
                                                      const void* v, void* out, int B, int H,
                                                      int Hkv, int Lq, int Lk, int d,
                                                      int causal, float sm_scale,
                                                      void* stream) {
  sage::set_last_launch_count(0);
  // --- arguments (host only; nothing touches the GPU before they pass)
  sage_status st = sage::check_shape(B, H, Hkv, Lq, Lk, d);
  if (st != SAGE_OK) return st;
  if ((st = sage::check_quant_len(Lk)) != SAGE_OK) return st;
  if (!q || !k || !v || !out) return SAGE_ERR_INVALID_ARG;
  if (!sage::aligned16(q) || !sage::aligned16(k) || !sage::aligned16(v) || !sage::aligned16(out))
    return SAGE_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;

  // --- scratch layout, each piece 256-byte aligned; reject what does not fit
  // (check_shape bounds every element count by 2^40, so no product wraps)
  const size_t nqb = (size_t)(Lq + 127) / 128, nkb = (size_t)(Lk + 63) / 64;
  const size_t off_q = 0;
  const size_t off_k = off_q + piece((size_t)B * H * Lq * d);
  const size_t off_qs = off_k + piece((size_t)B * Hkv * Lk * d);
  const size_t off_ks = off_qs + piece((size_t)B * H * nqb * sizeof(float));
  const size_t off_m = off_ks + piece((size_t)B * Hkv * nkb * sizeof(float));
  const size_t total = off_m + piece((size_t)B * Hkv * d * sizeof(float));
  if (total > kNoAllocScratchBytes) return SAGE_ERR_INVALID_ARG;

  // --- device: sm_100 only, then the scratch address
  if ((st = sage::check_device()) != SAGE_OK) return st;
  void* base = nullptr;
  if (scratch_on_current_device(&base) != cudaSuccess) return SAGE_ERR_CUDA;
  char* ws = static_cast<char*>(base);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int8_t* q_i8 = reinterpret_cast<int8_t*>(ws + off_q);
  int8_t* k_i8 = reinterpret_cast<int8_t*>(ws + off_k);
  float* q_scale = reinterpret_cast<float*>(ws + off_qs);
  float* k_scale = reinterpret_cast<float*>(ws + off_ks);
  float* k_mean = reinterpret_cast<float*>(ws + off_m);
  sage::QuantArgs qa{static_cast<const __half*>(q), static_cast<const __half*>(k), q_i8, k_i8,
                     q_scale, k_scale, k_mean, B, H, Hkv, Lq, Lk, d,
                     sage::fold_constant(sm_scale), SAGE_Q_BLOCK_ROWS};
  int launches = 0;
  cudaError_t e = sage::launch_quant(qa, s, &launches);
  if (e == cudaSuccess) {
    sage::AttnArgs aa{q_i8, k_i8, q_scale, k_scale, static_cast<const __half*>(v),
                      static_cast<__half*>(out), B, H, Hkv, Lq, Lk, d, causal == 1,
                      SAGE_Q_BLOCK_ROWS};
    e = sage::launch_attn(aa, s, &launches);
  }
  sage::set_last_launch_count(launches);
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}
