// api.cu — the extern "C" entry points of libspax.so: argument checks, plans and launches.
// Every entry point validates its arguments on the host and launches nothing on an error; see
// include/spax.h for the contract of each call.
#include <cmath>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace spax {

int sm_count_current_device() {
  static std::mutex mu;
  static std::unordered_map<int, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  cache[dev] = n;
  return n;
}

cudaError_t ensure_smem_limit(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::unordered_map<long long, int> done;  // (device, kernel) -> bytes already allowed
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const long long key = (static_cast<long long>(reinterpret_cast<uintptr_t>(kernel)) << 8) ^ dev;
  std::lock_guard<std::mutex> lk(mu);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  // always raise it: static shared memory counts against the 48 KB default too
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  done[key] = bytes;
  return cudaSuccess;
}

// Dynamic shared memory a masked GEMV may use (227 KB per CTA, less room for static variables).

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static spax_status launch_status(cudaError_t e) {
  if (e == cudaSuccess) return SPAX_OK;
  (void)cudaGetLastError();  // the error is reported through the status; clear the sticky-free one
  return SPAX_ERR_CUDA;
}

}  // namespace spax

using namespace spax;

extern "C" {

int spax_abi_version(void) { return SPAX_ABI_VERSION; }

const char* spax_status_string(int s) {
  switch (s) {
    case SPAX_OK: return "ok";
    case SPAX_ERR_ARG: return "invalid argument";
    case SPAX_ERR_SHAPE: return "unsupported shape";
    case SPAX_ERR_WORKSPACE: return "workspace missing or too small";
    case SPAX_ERR_CUDA: return "CUDA error";
    case SPAX_ERR_NONFINITE: return "non-finite input";
    case SPAX_ERR_TIMEOUT: return "pipeline wait timed out";
    case SPAX_ERR_INDEX: return "column count or index out of range";
    default: return "unknown status";
  }
}

size_t spax_pack_bytes(int d_out, int d_in, int full_fmt, size_t* full_bytes, size_t* approx_bytes) {
  if (d_out < 128 || d_out % 128 != 0 || d_in < 1) return 0;
  size_t f;
  if (full_fmt == SPAX_FULL_BF16)
    f = size_t(d_in) * d_out * 2;
  else if (full_fmt == SPAX_FULL_INT4_G128)
    f = size_t(d_in) * ((d_out + 1023) / 1024) * 528;
  else
    return 0;
  const size_t a = size_t(d_in) * ((d_out + 511) / 512) * 144;
  if (full_bytes) *full_bytes = f;
  if (approx_bytes) *approx_bytes = a;
  return f + a;
}

spax_status spax_pack_weights(const void* W, int d_out, int d_in, int full_fmt, void* full,
                              void* approx, void* stream) {
  if (!W || !full || !approx) return SPAX_ERR_ARG;
  if (full_fmt != SPAX_FULL_BF16 && full_fmt != SPAX_FULL_INT4_G128) return SPAX_ERR_ARG;
  if (d_out < 128 || d_out % 128 != 0 || d_in < 1) return SPAX_ERR_SHAPE;
  if (!aligned16(full) || !aligned16(approx) || (reinterpret_cast<uintptr_t>(W) & 1u))
    return SPAX_ERR_ARG;
  if (d_in > (1 << 30) / 32) return SPAX_ERR_SHAPE;
  return launch_status(launch_pack(W, d_out, d_in, full_fmt, full, approx,
                                   static_cast<cudaStream_t>(stream)));
}

spax_status spax_calibrate_thresholds(const float* calib_x, int n_tok, int d_in, int s_skip_bp,
                                      int s_below_full_bp, float* t_out, int32_t* status, void* ws,
                                      size_t ws_bytes, void* stream) {
  if (!calib_x || !t_out) return SPAX_ERR_ARG;
  if (n_tok < 1 || d_in < 1) return SPAX_ERR_SHAPE;
  const long long M = (long long)n_tok * d_in;
  if (M >= (1LL << 31)) return SPAX_ERR_SHAPE;
  if (s_skip_bp < 0 || s_skip_bp > 10000 || s_below_full_bp < 0 || s_below_full_bp > 10000)
    return SPAX_ERR_ARG;
  if (!ws || ws_bytes < calibrate_ws_bytes()) return SPAX_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return SPAX_ERR_ARG;
  auto qidx = [M](long long bp) {
    long long i = (bp * M + 5000) / 10000;
    return i > M - 1 ? M - 1 : i;
  };
  return launch_status(launch_calibrate(calib_x, M, qidx(s_skip_bp), qidx(s_below_full_bp), t_out,
                                        status, ws, static_cast<cudaStream_t>(stream)));
}

// The rule's parameters for d_in columns (shared by the mask and the masked GEMV).
static spax_status check_mask_params(const spax_mask_params& q, int d_in) {
  if (q.mode == SPAX_MASK_TOPK || q.mode == SPAX_MASK_TOPK_SCALED) {
    if (q.k_full < 0 || q.k_approx < 0 || (long long)q.k_full + q.k_approx > d_in)
      return SPAX_ERR_ARG;
  } else if (q.mode == SPAX_MASK_THRESHOLD || q.mode == SPAX_MASK_GUIDED) {
    if (!(q.t_skip >= 0.0f) || !(q.t_full >= q.t_skip)) return SPAX_ERR_ARG;  // rejects NaN too
    if (q.mode == SPAX_MASK_GUIDED) {
      if (q.s_skip_bp < 0 || q.s_below_full_bp < q.s_skip_bp || q.s_below_full_bp > 10000 ||
          q.delta_bp < 0 || q.delta_bp > 10000)
        return SPAX_ERR_ARG;
    }
  } else {
    return SPAX_ERR_ARG;
  }
  return SPAX_OK;
}

spax_status spax_build_mask(const float* x, int d_in, const spax_mask_params* p, uint8_t* tier,
                            int32_t* full_idx, int32_t* approx_idx, int32_t* counts,
                            int32_t* status, void* stream) {
  if (!x || !p || !tier || !full_idx || !approx_idx || !counts) return SPAX_ERR_ARG;
  if (d_in < 1 || d_in > SPAX_MASK_MAX_DIN) return SPAX_ERR_SHAPE;
  const spax_mask_params q = *p;
  const spax_status st = check_mask_params(q, d_in);
  if (st != SPAX_OK) return st;
  return launch_status(launch_mask(x, d_in, q, tier, full_idx, approx_idx, counts, status,
                                   static_cast<cudaStream_t>(stream)));
}

size_t spax_workspace_bytes(int op, int d_out, int d_in) {
  if (op == SPAX_OP_CALIBRATE) return calibrate_ws_bytes();
  if (op != SPAX_OP_TIERED_GEMV && op != SPAX_OP_DENSE_GEMV) return 0;
  // enough for either full-tier format
  GemvPlan pb, pi;
  const int sms = sm_count_current_device();
  const bool dense = op == SPAX_OP_DENSE_GEMV;
  if (!make_gemv_plan(d_out, d_in, SPAX_FULL_BF16, sms, dense, &pb)) return 0;
  if (!make_gemv_plan(d_out, d_in, SPAX_FULL_INT4_G128, sms, dense, &pi)) return 0;
  return pb.ws_bytes > pi.ws_bytes ? pb.ws_bytes : pi.ws_bytes;
}

spax_status spax_gemv_plan(int op, int d_out, int d_in, int full_fmt, int32_t* splits,
                           int32_t* row_tile) {
  if (op != SPAX_OP_TIERED_GEMV && op != SPAX_OP_DENSE_GEMV) return SPAX_ERR_ARG;
  GemvPlan pl;
  const int sms = sm_count_current_device();
  if (sms < 1) return SPAX_ERR_CUDA;
  if (!make_gemv_plan(d_out, d_in, full_fmt, sms, op == SPAX_OP_DENSE_GEMV, &pl)) return SPAX_ERR_SHAPE;
  if (splits) *splits = pl.S;
  if (row_tile) *row_tile = pl.R;
  return SPAX_OK;
}

spax_status spax_gemv_plan_sms(int op, int d_out, int d_in, int full_fmt, int sm_count,
                               int32_t* splits, int32_t* row_tile, size_t* ws_bytes) {
  if (op != SPAX_OP_TIERED_GEMV && op != SPAX_OP_DENSE_GEMV) return SPAX_ERR_ARG;
  if (sm_count < 1) return SPAX_ERR_ARG;
  GemvPlan pl;
  if (!make_gemv_plan(d_out, d_in, full_fmt, sm_count, op == SPAX_OP_DENSE_GEMV, &pl))
    return SPAX_ERR_SHAPE;
  if (splits) *splits = pl.S;
  if (row_tile) *row_tile = pl.R;
  if (ws_bytes) *ws_bytes = pl.ws_bytes;
  return SPAX_OK;
}

static spax_status gemv_common(const void* full, const void* approx, int full_fmt, const float* x,
                               const int32_t* fidx, const int32_t* aidx, const int32_t* counts,
                               float* y, int d_out, int d_in, int32_t* status, void* ws,
                               size_t ws_bytes, void* stream, bool dense,
                               unsigned long long wait_ns = 0, int drop_splits = 0) {
  if (!full || !x || !y) return SPAX_ERR_ARG;
  if (!dense && (!approx || !fidx || !aidx || !counts)) return SPAX_ERR_ARG;
  if (full_fmt != SPAX_FULL_BF16 && full_fmt != SPAX_FULL_INT4_G128) return SPAX_ERR_ARG;
  if (d_out < 128 || d_out % 128 != 0 || d_in < 1) return SPAX_ERR_SHAPE;
  if (!aligned16(full) || (!dense && !aligned16(approx)) || !aligned16(y)) return SPAX_ERR_ARG;
  const int sms = sm_count_current_device();
  if (sms < 1) return SPAX_ERR_CUDA;
  GemvPlan pl;
  if (!make_gemv_plan(d_out, d_in, full_fmt, sms, dense, &pl)) return SPAX_ERR_SHAPE;
  if (drop_splits && pl.S <= drop_splits) return SPAX_ERR_SHAPE;
  if (!ws || ws_bytes < pl.ws_bytes) return SPAX_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return SPAX_ERR_ARG;
  GemvLaunch a;
  a.wait_ns = wait_ns;
  a.drop_splits = drop_splits;
  a.full = full;
  a.approx = approx;
  a.x = x;
  a.full_idx = fidx;
  a.approx_idx = aidx;
  a.counts = counts;
  a.y = y;
  a.status = status;
  a.ws = ws;
  a.d_out = d_out;
  a.d_in = d_in;
  a.full_fmt = full_fmt;
  a.dense = dense;
  return launch_status(launch_gemv(a, pl, static_cast<cudaStream_t>(stream)));
}

spax_status spax_tiered_gemv(const spax_packed* W, const float* x, const int32_t* full_idx,
                             const int32_t* approx_idx, const int32_t* counts, float* y,
                             int32_t* status, void* ws, size_t ws_bytes, void* stream) {
  if (!W) return SPAX_ERR_ARG;
  return gemv_common(W->d_full, W->d_approx, W->full_fmt, x, full_idx, approx_idx, counts, y,
                     W->d_out, W->d_in, status, ws, ws_bytes, stream, false);
}

static spax_status masked_gemv_common(const spax_packed* W, const float* x, bool swiglu,
                                      float* x_out, const float* norms,
                                      const spax_mask_params* p, float* y,
                                      uint8_t* tier, int32_t* full_idx, int32_t* approx_idx,
                                      int32_t* counts, int32_t* status, void* ws, size_t ws_bytes,
                                      void* stream) {
  if (!W || !W->d_full || !W->d_approx || !x || !p || !y) return SPAX_ERR_ARG;
  if (W->full_fmt != SPAX_FULL_BF16 && W->full_fmt != SPAX_FULL_INT4_G128) return SPAX_ERR_ARG;
  if (W->d_out < 128 || W->d_out % 128 != 0 || W->d_in < 1) return SPAX_ERR_SHAPE;
  if (W->d_in > SPAX_MASK_MAX_DIN) return SPAX_ERR_SHAPE;
  if (!aligned16(W->d_full) || !aligned16(W->d_approx) || !aligned16(y)) return SPAX_ERR_ARG;
  const spax_mask_params q = *p;
  const spax_status st = check_mask_params(q, W->d_in);
  if (st != SPAX_OK) return st;
  const int sms = sm_count_current_device();
  if (sms < 1) return SPAX_ERR_CUDA;
  GemvPlan pl;
  if (!make_gemv_plan(W->d_out, W->d_in, W->full_fmt, sms, false, &pl)) return SPAX_ERR_SHAPE;
  if (masked_gemv_smem_bytes(pl, W->d_in) > kMaskedGemvSmemLimit) return SPAX_ERR_SHAPE;
  if (!ws || ws_bytes < pl.ws_bytes) return SPAX_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return SPAX_ERR_ARG;
  GemvLaunch a;
  a.full = W->d_full;
  a.approx = W->d_approx;
  a.x = x;
  a.full_idx = nullptr;
  a.approx_idx = nullptr;
  a.counts = nullptr;
  a.y = y;
  a.status = status;
  a.ws = ws;
  a.d_out = W->d_out;
  a.d_in = W->d_in;
  a.full_fmt = W->full_fmt;
  a.dense = false;
  return launch_status(launch_masked_gemv(a, q, swiglu, x_out, norms, tier, full_idx, approx_idx,
                                          counts, pl, static_cast<cudaStream_t>(stream)));
}

spax_status spax_masked_gemv(const spax_packed* W, const float* x, const spax_mask_params* p,
                             float* y, uint8_t* tier, int32_t* full_idx, int32_t* approx_idx,
                             int32_t* counts, int32_t* status, void* ws, size_t ws_bytes,
                             void* stream) {
  return masked_gemv_common(W, x, false, nullptr, nullptr, p, y, tier, full_idx, approx_idx, counts,
                            status, ws, ws_bytes, stream);
}

spax_status spax_masked_gemv_wina(const spax_packed* W, const float* x, const float* norms,
                                  const spax_mask_params* p, float* y, uint8_t* tier,
                                  int32_t* full_idx, int32_t* approx_idx, int32_t* counts,
                                  int32_t* status, void* ws, size_t ws_bytes, void* stream) {
  if (!norms) return SPAX_ERR_ARG;
  return masked_gemv_common(W, x, false, nullptr, norms, p, y, tier, full_idx, approx_idx, counts,
                            status, ws, ws_bytes, stream);
}

spax_status spax_output_change(const float* y, const float* y_ref, int n, double* acc,
                               void* stream) {
  if (!y || !y_ref || !acc) return SPAX_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(acc) & 7u) return SPAX_ERR_ARG;
  if (n < 1) return SPAX_ERR_SHAPE;
  return launch_status(launch_output_change(y, y_ref, n, acc, static_cast<cudaStream_t>(stream)));
}

spax_status spax_probe_sensitivity(const spax_packed* W, const float* X, int n_tok, int s_probe_bp,
                                   float* y2, double* acc, int32_t* status, void* ws,
                                   size_t ws_bytes, void* stream) {
  if (!W || !X || !y2 || !acc) return SPAX_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(acc) & 7u) return SPAX_ERR_ARG;
  if (n_tok < 1) return SPAX_ERR_SHAPE;
  if (s_probe_bp < 0 || s_probe_bp > 10000) return SPAX_ERR_ARG;
  const int d = W->d_in, d_out = W->d_out;
  const int skip = (int)(((long long)s_probe_bp * d + 5000) / 10000);
  spax_mask_params all = {}, probe = {};
  all.mode = probe.mode = SPAX_MASK_TOPK;
  all.k_full = d;                 // the reference: every column in full
  probe.k_full = d - skip;        // the probe: the skip smallest |x| left out, the rest in full
  float* y_ref = y2;
  float* y = y2 + d_out;
  if (reinterpret_cast<uintptr_t>(y) & 15u) return SPAX_ERR_ARG;
  for (int t = 0; t < n_tok; ++t) {
    const float* x = X + (size_t)t * d;
    spax_status st = masked_gemv_common(W, x, false, nullptr, nullptr, &all, y_ref, nullptr,
                                        nullptr, nullptr, nullptr, status, ws, ws_bytes, stream);
    if (st != SPAX_OK) return st;
    st = masked_gemv_common(W, x, false, nullptr, nullptr, &probe, y, nullptr, nullptr, nullptr,
                            nullptr, status, ws, ws_bytes, stream);
    if (st != SPAX_OK) return st;
    st = launch_status(launch_output_change(y, y_ref, d_out, acc, static_cast<cudaStream_t>(stream)));
    if (st != SPAX_OK) return st;
  }
  return SPAX_OK;
}

spax_status spax_column_norms(const void* W, int d_out, int d_in, float* norms, void* stream) {
  if (!W || !norms) return SPAX_ERR_ARG;
  if (d_out < 1 || d_in < 1) return SPAX_ERR_SHAPE;
  return launch_status(launch_column_norms(W, d_out, d_in, norms, static_cast<cudaStream_t>(stream)));
}

spax_status spax_masked_gemv_swiglu(const spax_packed* W, const float* gu,
                                    const spax_mask_params* p, float* y, float* x_out,
                                    uint8_t* tier, int32_t* full_idx, int32_t* approx_idx,
                                    int32_t* counts, int32_t* status, void* ws, size_t ws_bytes,
                                    void* stream) {
  return masked_gemv_common(W, gu, true, x_out, nullptr, p, y, tier, full_idx, approx_idx, counts,
                            status, ws, ws_bytes, stream);
}

spax_status spax_test_tiered_gemv_timeout(const spax_packed* W, const float* x,
                                          const int32_t* full_idx, const int32_t* approx_idx,
                                          const int32_t* counts, float* y, int32_t* status,
                                          void* ws, size_t ws_bytes, uint64_t wait_limit_ns,
                                          void* stream) {
  if (!W) return SPAX_ERR_ARG;
  if (wait_limit_ns < 1000000ull || wait_limit_ns > 2000000000ull) return SPAX_ERR_ARG;
  if (!ws) {  // the fixed scratch array of spax_tiered_gemv_fixed_scratch
    ws = fixed_scratch_current_device_ptr(&ws_bytes);
    if (!ws) return SPAX_ERR_CUDA;
  }
  return gemv_common(W->d_full, W->d_approx, W->full_fmt, x, full_idx, approx_idx, counts, y,
                     W->d_out, W->d_in, status, ws, ws_bytes, stream, false, wait_limit_ns, 1);
}

spax_status spax_dense_gemv(const void* Wt, const float* x, float* y, int d_out, int d_in,
                            int32_t* status, void* ws, size_t ws_bytes, void* stream) {
  return gemv_common(Wt, nullptr, SPAX_FULL_BF16, x, nullptr, nullptr, nullptr, y, d_out, d_in,
                     status, ws, ws_bytes, stream, true);
}

// Bisection on the mean-restoring shift c (the mean of the clamped budgets is continuous and
// non-decreasing in c); 200 halvings reach the fp64 resolution of the bracket.
spax_status spax_block_budgets(const double* sens, int n, double s, double lambda, double lo,
                               double hi, double* out) {
  if (!sens || !out || n < 1) return SPAX_ERR_ARG;
  if (!(lo >= 0.0 && lo <= s && s <= hi && hi <= 1.0) || !(lambda >= 0.0)) return SPAX_ERR_ARG;
  double sbar = 0.0;
  for (int b = 0; b < n; ++b) {
    if (!(sens[b] > 0.0) || !std::isfinite(sens[b])) return SPAX_ERR_ARG;
    sbar += sens[b];
  }
  sbar /= n;
  double amin = 1e300, amax = -1e300;
  for (int b = 0; b < n; ++b) {
    const double a = s * (1.0 - lambda * (sens[b] / sbar - 1.0));
    out[b] = a;
    amin = a < amin ? a : amin;
    amax = a > amax ? a : amax;
  }
  auto mean_at = [&](double c) {
    double m = 0.0;
    for (int b = 0; b < n; ++b) {
      double v = out[b] + c;
      m += v < lo ? lo : (v > hi ? hi : v);
    }
    return m / n;
  };
  double c = 0.0;
  if (mean_at(0.0) != s) {
    double cl = lo - amax, ch = hi - amin;  // mean(cl) = lo <= s <= hi = mean(ch)
    for (int it = 0; it < 200; ++it) {
      const double mid = 0.5 * (cl + ch);
      if (mean_at(mid) < s)
        cl = mid;
      else
        ch = mid;
    }
    c = 0.5 * (cl + ch);
  }
  for (int b = 0; b < n; ++b) {
    const double v = out[b] + c;
    out[b] = v < lo ? lo : (v > hi ? hi : v);
  }
  return SPAX_OK;
}

spax_status spax_greedy_allocation(const double* f, int n, double alpha, double p_target,
                                   double p_max, spax_block_error_fn err, void* ctx,
                                   int max_steps, double* p_out, int32_t* order,
                                   int32_t* steps) {
  if (!f || !p_out || !steps || !err || n < 1 || max_steps < 0) return SPAX_ERR_ARG;
  if (!(alpha > 0.0) || !(p_target >= 0.0) || !(p_target <= p_max) || !(p_max <= 1.0))
    return SPAX_ERR_ARG;
  double fsum = 0.0;
  for (int m = 0; m < n; ++m) {
    if (!(f[m] > 0.0) || !std::isfinite(f[m])) return SPAX_ERR_ARG;
    fsum += f[m];
  }
  const double fbar = fsum / n;
  std::vector<double> p(n, 0.0), cand(n);
  *steps = 0;
  spax_status st = SPAX_OK;
  for (;;) {
    double P = 0.0;
    for (int m = 0; m < n; ++m) P += f[m] * p[m];
    if (P / fsum >= p_target - 1e-12) break;
    if (*steps >= max_steps) {
      st = SPAX_ERR_ARG;
      break;
    }
    int best = -1;
    double best_err = 0.0;
    for (int m = 0; m < n; ++m) {
      const double step = alpha * fbar / f[m];
      if (p[m] + step > p_max + 1e-12) continue;
      cand = p;
      cand[m] += step;
      const double e = err(cand.data(), n, ctx);
      if (best < 0 || e < best_err) {
        best = m;
        best_err = e;
      }
    }
    if (best < 0) {  // every matrix is at its ceiling
      st = SPAX_ERR_ARG;
      break;
    }
    p[best] += alpha * fbar / f[best];
    if (order) order[*steps] = best;
    ++*steps;
  }
  for (int m = 0; m < n; ++m) p_out[m] = p[m];
  return st;
}

uint64_t spax_weight_bytes(int d_out, int full_fmt, int64_t n_full, int64_t n_approx) {
  if (d_out < 128 || d_out % 128 != 0 || n_full < 0 || n_approx < 0) return 0;
  const uint64_t groups = uint64_t(d_out) / 128;
  uint64_t pf;
  if (full_fmt == SPAX_FULL_BF16)
    pf = 2ull * d_out;
  else if (full_fmt == SPAX_FULL_INT4_G128)
    pf = uint64_t(d_out) / 2 + 2 * groups;
  else
    return 0;
  const uint64_t pa = uint64_t(d_out) / 4 + 4 * groups;
  return uint64_t(n_full) * pf + uint64_t(n_approx) * pa;
}

}  // extern "C"
