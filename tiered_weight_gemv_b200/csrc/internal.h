// internal.h — host-side declarations shared by the libspax translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/spax.h"

namespace spax {

// Split-K plan of one GEMV launch: grid (T row tiles of R rows) x (S column splits), one wave
// (T * S <= SMs whenever S > 1). The S flagged partial rows of a tile live at off_part in the
// workspace ([S][d_out] 64-bit words, zero at rest); ws_bytes is the workspace the launch needs.
struct GemvPlan {
  int R, T, S;
  size_t off_part, ws_bytes;
};

int sm_count_current_device();  // cached per device; 0 on error
// dense: the plan of the dense GEMV (its own row-tile rule); otherwise the tiered kernels'.
bool make_gemv_plan(int d_out, int d_in, int full_fmt, int sm_count, bool dense, GemvPlan* plan);

struct GemvLaunch {
  const void* full;
  const void* approx;
  const float* x;
  const int32_t* full_idx;
  const int32_t* approx_idx;
  const int32_t* counts;
  float* y;
  int32_t* status;
  void* ws;
  int d_out, d_in, full_fmt;
  bool dense;
  unsigned long long wait_ns = 0;  // bound of the split-K wait (0: kWaitLimitNs)
  int drop_splits = 0;  // failure-detection test only: launch the last drop_splits splits of no tile
};
cudaError_t launch_gemv(const GemvLaunch& a, const GemvPlan& plan, cudaStream_t stream);
// The mask and the GEMV in one launch (every CTA computes the token's lists itself); the tier,
// list and count outputs may be null. Shared memory it needs for a plan and d_in.
// swiglu: a.x holds [g; u] (2 * d_in) and x_j = silu(g_j) * u_j (written to x_out when set).
// norms (may be null): rank columns by the WINA score |x_j| * norms[j] instead of |x_j|.
cudaError_t launch_masked_gemv(const GemvLaunch& a, const spax_mask_params& prm, bool swiglu,
                               float* x_out, const float* norms, uint8_t* tier, int32_t* full_idx,
                               int32_t* approx_idx, int32_t* counts, const GemvPlan& plan,
                               cudaStream_t stream);
size_t masked_gemv_smem_bytes(const GemvPlan& plan, int d_in);
// Dynamic shared memory a masked GEMV may take (227 KB per CTA, less room for static shared).
constexpr size_t kMaskedGemvSmemLimit = 227 * 1024 - 1024;

cudaError_t launch_mask(const float* x, int d_in, const spax_mask_params& p, uint8_t* tier,
                        int32_t* full_idx, int32_t* approx_idx, int32_t* counts, int32_t* status,
                        cudaStream_t stream);

cudaError_t launch_pack(const void* W, int d_out, int d_in, int full_fmt, void* full, void* approx,
                        cudaStream_t stream);
cudaError_t launch_column_norms(const void* W, int d_out, int d_in, float* norms,
                                cudaStream_t stream);

// The fixed scratch array of spax_tiered_gemv_fixed_scratch on the current device (nullptr if
// its address could not be looked up); *bytes gets its size.
uint8_t* fixed_scratch_current_device_ptr(size_t* bytes);

size_t calibrate_ws_bytes();
cudaError_t launch_output_change(const float* y, const float* y_ref, int n, double* acc,
                                 cudaStream_t stream);
cudaError_t launch_calibrate(const float* X, long long M, long long idx_skip, long long idx_full,
                             float* t_out, int32_t* status, void* ws, cudaStream_t stream);

// Launch helper: every libspax kernel is launched as a programmatic dependent of its
// predecessor in the stream (it calls griddepcontrol.wait before touching global memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Raise a kernel's dynamic shared-memory limit once per device.
cudaError_t ensure_smem_limit(const void* kernel, int bytes);

}  // namespace spax
