// noalloc.cu — spax_tiered_gemv_fixed_scratch: the tiered GEMV with its split-K scratch in a
// fixed device array that is part of the library image, so the call allocates nothing and needs
// no workspace argument.
//
// Who needs it: callers that cannot allocate device memory at the point of the call — code that
// runs inside an allocator-free region of a larger runtime (for instance a custom allocator's
// own callbacks, or a plugin of a host that owns every device allocation and hands out none),
// and callers that must not make the allocator synchronise the device. The regular entry point
// needs a caller-owned workspace; this one does not.
//
// Scratch layout (kFixedScratchBytes in total, 256-byte aligned): the flagged split-K partial
// sums of the launch's plan from offset 0. A word is zero until a split publishes its value (the
// value's bits and a ready flag in one 64-bit store); the CTA that sums it clears it again. Device
// globals start at zero when the library's module loads and every completed call leaves the
// words it used at zero, so calls of any shape find a clean array.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace spax {

constexpr size_t kFixedScratchBytes = size_t(4) << 20;  // 4 MiB per device

static __device__ __align__(256) uint8_t g_fixed_scratch[kFixedScratchBytes];

// Driver calls the address cache needs, resolved through the runtime (no link-time dependency on
// the driver library): the current context and its process-unique id.
using CtxGetCurrentFn = int (*)(void** ctx);                       // cuCtxGetCurrent
using CtxGetIdFn = int (*)(void* ctx, unsigned long long* id);     // cuCtxGetId

// Id of the context current on this thread; false when there is none (or the driver lacks the
// call), in which case the caller looks the address up again on every call.
static bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
    (void)cudaGetLastError();
  });
  if (!get_current || !get_id) return false;
  void* ctx = nullptr;
  if (get_current(&ctx) != 0 || !ctx) return false;
  return get_id(ctx, id) == 0;
}

// Device address of g_fixed_scratch in the current device's context; nullptr if the lookup
// failed. It is looked up (cudaGetSymbolAddress, with that device current) the first time a
// device's context calls in, and again whenever that device's context has changed since (a
// cudaDeviceReset makes a new context, whose copy of the library's module is a new array, zero
// again). Contexts are told apart by their process-unique id, not by handle.
static uint8_t* fixed_scratch_current_device() {
  constexpr int kMaxDevices = 64;
  struct Entry {
    unsigned long long ctx_id;
    uint8_t* addr;
  };
  static std::mutex mu;
  static Entry cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return nullptr;
  }
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lk(mu);
  if (have_id && cache[dev].addr && cache[dev].ctx_id == id) return cache[dev].addr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_fixed_scratch) != cudaSuccess || !p) {
    (void)cudaGetLastError();
    return nullptr;
  }
  if (!have_id) have_id = current_context_id(&id);  // the lookup made the context current
  cache[dev].addr = static_cast<uint8_t*>(p);
  cache[dev].ctx_id = have_id ? id : 0;  // id 0 is never a context's: the next call looks again
  return cache[dev].addr;
}

uint8_t* fixed_scratch_current_device_ptr(size_t* bytes) {
  if (bytes) *bytes = kFixedScratchBytes;
  return fixed_scratch_current_device();
}

}  // namespace spax

using namespace spax;

extern "C" {

size_t spax_fixed_scratch_bytes(void) { return kFixedScratchBytes; }

spax_status spax_fixed_scratch_reset(void* stream) {
  uint8_t* scratch = fixed_scratch_current_device();
  if (!scratch) return SPAX_ERR_CUDA;
  if (cudaMemsetAsync(scratch, 0, kFixedScratchBytes, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return SPAX_ERR_CUDA;
  }
  return SPAX_OK;
}

spax_status spax_tiered_gemv_fixed_scratch(const spax_packed* W, const float* x,
                                           const int32_t* full_idx, const int32_t* approx_idx,
                                           const int32_t* counts, float* y, int32_t* status,
                                           void* stream) {
  if (!W || !W->d_full || !W->d_approx || !x || !y || !full_idx || !approx_idx || !counts)
    return SPAX_ERR_ARG;
  if (W->full_fmt != SPAX_FULL_BF16 && W->full_fmt != SPAX_FULL_INT4_G128) return SPAX_ERR_ARG;
  if (W->d_out < 128 || W->d_out % 128 != 0 || W->d_in < 1) return SPAX_ERR_SHAPE;
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(W->d_full) || !a16(W->d_approx) || !a16(y)) return SPAX_ERR_ARG;
  const int sms = sm_count_current_device();
  if (sms < 1) return SPAX_ERR_CUDA;
  GemvPlan pl;
  if (!make_gemv_plan(W->d_out, W->d_in, W->full_fmt, sms, false, &pl)) return SPAX_ERR_SHAPE;
  if (pl.ws_bytes > kFixedScratchBytes) return SPAX_ERR_WORKSPACE;  // see spax_gemv_plan_sms
  uint8_t* scratch = fixed_scratch_current_device();
  if (!scratch) return SPAX_ERR_CUDA;
  GemvLaunch a;
  a.full = W->d_full;
  a.approx = W->d_approx;
  a.x = x;
  a.full_idx = full_idx;
  a.approx_idx = approx_idx;
  a.counts = counts;
  a.y = y;
  a.status = status;
  a.ws = scratch;
  a.d_out = W->d_out;
  a.d_in = W->d_in;
  a.full_fmt = W->full_fmt;
  a.dense = false;
  const cudaError_t e = launch_gemv(a, pl, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return SPAX_ERR_CUDA;
  }
  return SPAX_OK;
}

}  // extern "C"
