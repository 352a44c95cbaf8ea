// common.cuh — device helpers shared by the libspax kernels (sm_100a only).
//
// Thin wrappers over PTX: the global timer that bounds every wait, programmatic dependent
// launch, shared-memory vector loads, packed fp32x2 FMA, and the bf16 bit tricks the GEMV inner
// loops use.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/spax.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libspax targets sm_100a (B200) only"
#endif

namespace spax {

// Default bound of a wait on another CTA's data before the kernel reports SPAX_ERR_TIMEOUT.
constexpr unsigned long long kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- programmatic dependent launch ------------------------------------------------------
// Wait until the preceding grid in the stream has completed and its writes are visible (a
// no-op when the kernel was not launched as a programmatic dependent).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next grid in the stream to start launching (it still waits for our completion).
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- shared-memory vector loads ---------------------------------------------------------------
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}

// ---- packed fp32x2 FMA (sm_100): d = a * b + c, two lanes per instruction -----------------------
struct f2 {
  float x, y;
};
__device__ __forceinline__ f2 ffma2(f2 a, f2 b, f2 c) {
  unsigned long long ra, rb, rc, rd;
  ra = (static_cast<unsigned long long>(__float_as_uint(a.y)) << 32) | __float_as_uint(a.x);
  rb = (static_cast<unsigned long long>(__float_as_uint(b.y)) << 32) | __float_as_uint(b.x);
  rc = (static_cast<unsigned long long>(__float_as_uint(c.y)) << 32) | __float_as_uint(c.x);
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  f2 d;
  d.x = __uint_as_float(static_cast<uint32_t>(rd));
  d.y = __uint_as_float(static_cast<uint32_t>(rd >> 32));
  return d;
}

// bf16 pair in one 32-bit word -> the two fp32 values (exact: bf16 is the top half of fp32).
// The low half moves up by a multiply, which the compiler may issue on the FMA pipe and so
// leave the integer pipe to the decoding of the small formats.
__device__ __forceinline__ f2 bf16x2_to_f2(uint32_t w) {
  f2 r;
  r.x = __uint_as_float(w * 65536u);
  r.y = __uint_as_float(w & 0xFFFF0000u);
  return r;
}

// Gated-MLP activation x = silu(g) * u, silu(g) = g / (1 + e^-g), in fp32 with each step rounded
// on its own (no contraction): the one definition every use of x in a kernel goes through.
__device__ __forceinline__ float swiglu_x(float g, float u) {
  return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))), u);
}

__device__ __forceinline__ void record_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

}  // namespace spax
