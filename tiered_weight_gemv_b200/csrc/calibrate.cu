// calibrate.cu — quantile thresholds of pooled |x| over calibration tokens.
//
// Source: TopK-Guided (arXiv 2610.01763), §2.1 — each token's natural sparsity is estimated
// from a calibrated threshold; §2.2 — a calibration pass over held-out tokens.
// t(s) = the order statistic of 0-based rank idx = min(floor(s*M + 1/2), M - 1) of the M
// ascending values |x| (idx computed on the host in integer arithmetic).
//
// Radix select on the fp32 bit pattern of |x| (sign cleared: monotone as an unsigned integer),
// three passes of 11/11/9 bits, both thresholds at once. Each pass: a grid-wide histogram of the
// candidates that match the prefix found so far (shared-memory histograms merged with global
// atomics), then a one-CTA step that picks the bin holding the target rank.
#include "common.cuh"
#include "internal.h"

namespace spax {

struct CalibState {
  uint32_t prefix[2];  // key bits fixed so far
  uint32_t rem[2];     // 1-based rank still to find among the matching keys
};

constexpr int kCalibThreads = 512;

size_t calibrate_ws_bytes() { return 256 + 2 * 2048 * sizeof(uint32_t); }

__global__ void calib_init_kernel(CalibState* st, uint32_t* hist, long long idx_skip,
                                  long long idx_full) {
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    st->prefix[0] = st->prefix[1] = 0u;
    st->rem[0] = (uint32_t)(idx_skip + 1);
    st->rem[1] = (uint32_t)(idx_full + 1);
  }
  for (int i = threadIdx.x; i < 2 * 2048; i += blockDim.x) hist[i] = 0u;
}

__global__ void __launch_bounds__(kCalibThreads)
    calib_hist_kernel(const float* __restrict__ X, long long M, const CalibState* st,
                      uint32_t* hist, int shift, int nbits, int32_t* status) {
  __shared__ uint32_t h[2][2048];
  pdl_wait();
  pdl_launch_dependents();
  const int nb = 1 << nbits, hs = shift + nbits;
  for (int i = threadIdx.x; i < 2 * 2048; i += blockDim.x) (&h[0][0])[i] = 0u;
  const uint32_t p0 = st->prefix[0] >> hs, p1 = st->prefix[1] >> hs;
  __syncthreads();
  int bad = 0;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < M;
       i += (long long)gridDim.x * blockDim.x) {
    const uint32_t k = __float_as_uint(__ldg(X + i)) & 0x7FFFFFFFu;
    bad |= k >= 0x7F800000u;
    const uint32_t d = (k >> shift) & (nb - 1);
    if ((k >> hs) == p0) atomicAdd(&h[0][d], 1u);
    if ((k >> hs) == p1) atomicAdd(&h[1][d], 1u);
  }
  if (bad) record_status(status, SPAX_ERR_NONFINITE);
  __syncthreads();
  for (int i = threadIdx.x; i < 2 * nb; i += blockDim.x) {
    const int t = i / nb, b = i % nb;
    const uint32_t v = h[t][b];
    if (v) atomicAdd(&hist[t * 2048 + b], v);
  }
}

// One CTA: for each target, the bin b (ascending) with below(b) < rem <= below(b) + hist[b].
__global__ void __launch_bounds__(1024)
    calib_select_kernel(CalibState* st, uint32_t* hist, int shift, int nbits, float* t_out,
                        int last) {
  __shared__ uint32_t s_warp[2][32];
  __shared__ uint32_t s_bin[2], s_rem[2];
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nb = 1 << nbits;
  const uint32_t rem0 = st->rem[0], rem1 = st->rem[1];
  // thread i owns bins 2i, 2i+1 (ascending)
  for (int t = 0; t < 2; ++t) {
    const uint32_t rem = t ? rem1 : rem0;
    const int b0 = 2 * tid, b1 = 2 * tid + 1;
    const uint32_t h0 = b0 < nb ? hist[t * 2048 + b0] : 0u, h1 = b1 < nb ? hist[t * 2048 + b1] : 0u;
    // exclusive scan of h0 + h1 across the CTA (counts fit in 32 bits: M < 2^31)
    uint32_t v = h0 + h1, incl = v;
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) s_warp[t][warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const uint32_t w = s_warp[t][lane];
      uint32_t wi = w;
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += n;
      }
      s_warp[t][lane] = wi - w;
    }
    __syncthreads();
    const uint32_t below = s_warp[t][warp] + incl - v;
    if (below < rem && rem <= below + h0) {
      s_bin[t] = (uint32_t)b0;
      s_rem[t] = rem - below;
    } else if (below + h0 < rem && rem <= below + h0 + h1) {
      s_bin[t] = (uint32_t)b1;
      s_rem[t] = rem - below - h0;
    }
    __syncthreads();
  }
  for (int i = tid; i < 2 * 2048; i += blockDim.x) hist[i] = 0u;
  if (tid == 0) {
    for (int t = 0; t < 2; ++t) {
      st->prefix[t] |= s_bin[t] << shift;
      st->rem[t] = s_rem[t];
      if (last) t_out[t] = __uint_as_float(st->prefix[t]);
    }
  }
}

cudaError_t launch_calibrate(const float* X, long long M, long long idx_skip, long long idx_full,
                             float* t_out, int32_t* status, void* ws, cudaStream_t stream) {
  auto* st = static_cast<CalibState*>(ws);
  auto* hist = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + 256);
  cudaError_t e = launch_pdl(calib_init_kernel, dim3(1), dim3(256), 0, stream, st, hist, idx_skip,
                             idx_full);
  if (e != cudaSuccess) return e;
  const int shifts[3] = {20, 9, 0}, nbits[3] = {11, 11, 9};
  const int sms = sm_count_current_device();
  long long blocks = (M + kCalibThreads * 8 - 1) / (kCalibThreads * 8);
  const long long cap = (long long)(sms > 0 ? sms : 148) * 4;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  for (int pass = 0; pass < 3; ++pass) {
    e = launch_pdl(calib_hist_kernel, dim3((unsigned)blocks), dim3(kCalibThreads), 0, stream, X, M,
                   static_cast<const CalibState*>(st), hist, shifts[pass], nbits[pass], status);
    if (e != cudaSuccess) return e;
    e = launch_pdl(calib_select_kernel, dim3(1), dim3(1024), 0, stream, st, hist, shifts[pass],
                   nbits[pass], t_out, pass == 2 ? 1 : 0);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ---- output change of a sparsified projection (the sensitivity probe) -------------------------
// acc[0] += Σ_i (y_i - y_ref_i)^2, acc[1] += Σ_i y_ref_i^2 in fp64, by one CTA in a fixed order
// (strided per-thread sums, then a fixed tree), so the result does not depend on timing.
constexpr int kChangeThreads = 512;

__global__ void __launch_bounds__(kChangeThreads)
    output_change_kernel(const float* __restrict__ y, const float* __restrict__ y_ref, int n,
                         double* acc) {
  __shared__ double s0[kChangeThreads / 32], s1[kChangeThreads / 32];
  pdl_wait();
  pdl_launch_dependents();
  double a = 0.0, b = 0.0;
  for (int i = threadIdx.x; i < n; i += kChangeThreads) {
    const double r = (double)y_ref[i], e = (double)y[i] - r;
    a = fma(e, e, a);
    b = fma(r, r, b);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) s0[wid] = a, s1[wid] = b;
  __syncthreads();
  if (threadIdx.x == 0) {
    double ta = 0.0, tb = 0.0;
    for (int w = 0; w < kChangeThreads / 32; ++w) ta += s0[w], tb += s1[w];
    acc[0] += ta;
    acc[1] += tb;
  }
}

cudaError_t launch_output_change(const float* y, const float* y_ref, int n, double* acc,
                                 cudaStream_t stream) {
  return launch_pdl(output_change_kernel, dim3(1), dim3(kChangeThreads), 0, stream, y, y_ref, n,
                    acc);
}

}  // namespace spax
