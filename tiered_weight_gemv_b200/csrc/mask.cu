// mask.cu — per-token tier of every column and the compacted column lists (one CTA).
//
// Sources: SpAx (arXiv 2610.02598), Abstract — skip the columns whose activations are closest
// to zero, approximate the smaller ones, read the largest in full. TopK-Guided (arXiv
// 2610.01763), Abstract and §1 — the threshold rule (TEAL) and the fixed-count TopK rule
// (WINA); §2.1 — the natural sparsity estimated from the calibrated threshold, clipped to a ±δ
// band around the target, then TopK; mask construction is O(d).
//
// Rank order: larger |x| first; equal |x| by lower column index first. |x| is handled as its
// fp32 bit pattern with the sign cleared (monotone as an unsigned integer for finite values,
// and -0.0 == +0.0).
//
// Selecting the K-th largest key (both boundaries, K1 = #full and K2 = #full + #approx):
//   fast path: one pass of shared-memory atomics into a coarse histogram (the key's exponent,
//   256 bins) and a fine one (exponent and 7 mantissa bits, 32768 16-bit bins). One warp per
//   boundary scans the coarse bins and then the 128 fine bins under the chosen coarse bin with
//   shuffles; the few keys of the boundary fine bin (tens for Laplace-like activations) are then
//   ranked exactly against each other (key, then column);
//   fallback (a boundary bin holding more than kCandCap keys, i.e. many equal or near-equal |x|):
//   a three-pass 11/11/9-bit radix select; ties at the boundary key are resolved by an ordered
//   count of equal keys.
// Every pass over the columns is strided (thread t takes t, t+512, ...: conflict-free shared
// memory, coalesced global memory, independent iterations). Ordered results (the ascending
// column lists, the equal-key ranks) come from warp segments: warp w owns a contiguous run of
// columns, counts with ballots, and one small scan over the 16 warps gives every warp its
// offset; the lists are then written directly with coalesced stores.
#include "common.cuh"
#include "internal.h"

namespace spax {

constexpr int kMaskThreads = 512;
constexpr int kMaskWarps = kMaskThreads / 32;
constexpr int kFineWords = 16384;  // 32768 bins of 16 bits, two per word
constexpr int kCoarseBins = 256;
constexpr int kCandCap = 512;      // boundary keys ranked by brute force per target

// Exclusive scan of one value per warp (called by all threads; lane 0 of each warp supplies v).
// Returns the warp's offset to every lane; *total gets the sum.
__device__ __forceinline__ uint32_t warps_excl_scan(uint32_t v, uint32_t* s_warp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = lane < kMaskWarps ? s_warp[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < kMaskWarps) s_warp[16 + lane] = wi - w;
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  return s_warp[16 + warp];
}

// Block-wide sum (all threads call; result on every thread).
__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* s_warp, uint32_t* total) {
  v = __reduce_add_sync(0xffffffffu, v);
  (void)warps_excl_scan(v, s_warp, total);
  return *total;
}

// One warp: the first position, scanning PER consecutive counts per lane from the top (lane 0
// owns the highest entries), at which the running count from the top reaches K. Counts are
// given by get(i), i = 0 the highest. Returns the index and the count strictly above it.
template <int PER, typename Get>
__device__ __forceinline__ void warp_find_from_top(uint32_t K, uint32_t above0, Get get, int* idx,
                                                   uint32_t* above) {
  const int lane = threadIdx.x & 31;
  uint32_t c[PER], tot = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    c[i] = get(lane * PER + i);
    tot += c[i];
  }
  uint32_t incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  uint32_t cum = above0 + incl - tot;
  int found = -1;
  uint32_t fa = 0;
  if (cum < K && K <= cum + tot) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      if (found < 0 && cum + c[i] >= K) {
        found = lane * PER + i;
        fa = cum;
      }
      cum += c[i];
    }
  }
  const uint32_t ball = __ballot_sync(0xffffffffu, found >= 0);
  const int src = ball ? __ffs(ball) - 1 : 0;
  *idx = __shfl_sync(0xffffffffu, found, src);
  *above = __shfl_sync(0xffffffffu, fa, src);
}

// Band clip of TopK-Guided §2.1 in integer basis points: m = min(max(n, lo), hi) with
// lo = ceil((s - δ) d), hi = min(floor((s + δ) d), d).
__device__ __forceinline__ long long guided_clip(long long n, long long d, long long s_bp,
                                                 long long delta_bp) {
  const long long lo_num = (s_bp - delta_bp) * d;
  const long long lo = lo_num <= 0 ? 0 : (lo_num + 9999) / 10000;
  long long hi = (s_bp + delta_bp) * d / 10000;
  if (hi > d) hi = d;
  long long m = n < lo ? lo : n;
  if (m > hi) m = hi;
  return m;
}

size_t mask_smem_bytes(int d) {
  const size_t dpad = (size_t(d) + 15) & ~size_t(15);
  return dpad * 4 + dpad + size_t(kFineWords + kCoarseBins) * 4;
}

__global__ void __launch_bounds__(kMaskThreads, 1)
    mask_kernel(const float* __restrict__ x, int d, spax_mask_params prm, uint8_t* __restrict__ tier,
                int32_t* __restrict__ full_idx, int32_t* __restrict__ approx_idx,
                int32_t* __restrict__ counts, int32_t* status) {
  extern __shared__ __align__(16) uint32_t dyn[];
  const int dpad = (d + 15) & ~15;
  uint32_t* __restrict__ keys = dyn;                                      // [dpad]
  uint8_t* __restrict__ flags = reinterpret_cast<uint8_t*>(dyn + dpad);  // [dpad]
  uint32_t* fine = dyn + dpad + dpad / 4;  // [kFineWords]; later the candidates / radix bins
  uint32_t* coarse = fine + kFineWords;    // [kCoarseBins]
  __shared__ uint32_t s_warp[32];
  __shared__ uint32_t s_total;
  __shared__ uint32_t s_bin[2], s_above[2], s_cc[2], s_sel_bin[2], s_sel_rem[2];

  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  pdl_wait();
  pdl_launch_dependents();

  // ---- keys = |x| bits (vector loads when x is 16-byte aligned); NaN/Inf is an error ----
  if (tid < 2) s_cc[tid] = 0u;
  int bad = 0;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) == 0) {
    const int d4 = d >> 2;
    for (int i = tid; i < d4; i += kMaskThreads) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(x) + i);
      const uint4 k = make_uint4(v.x & 0x7FFFFFFFu, v.y & 0x7FFFFFFFu, v.z & 0x7FFFFFFFu,
                                 v.w & 0x7FFFFFFFu);
      bad |= (k.x >= 0x7F800000u) | (k.y >= 0x7F800000u) | (k.z >= 0x7F800000u) |
             (k.w >= 0x7F800000u);
      reinterpret_cast<uint4*>(keys)[i] = k;
    }
    for (int j = 4 * d4 + tid; j < d; j += kMaskThreads) {
      const uint32_t k = __float_as_uint(__ldg(x + j)) & 0x7FFFFFFFu;
      bad |= (k >= 0x7F800000u);
      keys[j] = k;
    }
  } else {
    for (int j = tid; j < d; j += kMaskThreads) {
      const uint32_t k = __float_as_uint(__ldg(x + j)) & 0x7FFFFFFFu;
      bad |= (k >= 0x7F800000u);
      keys[j] = k;
    }
  }
  for (int i = tid; i < dpad / 4; i += kMaskThreads) reinterpret_cast<uint32_t*>(flags)[i] = 0u;
  if (__syncthreads_or(bad)) {
    for (int j = tid; j < d; j += kMaskThreads) tier[j] = 0;
    if (tid == 0) {
      counts[0] = counts[1] = counts[2] = counts[3] = 0;
      record_status(status, SPAX_ERR_NONFINITE);
    }
    return;
  }

  // ---- natural counts of the threshold rule ----
  uint32_t n1 = 0, n2 = 0;
  const uint32_t ts = __float_as_uint(prm.t_skip) & 0x7FFFFFFFu;
  const uint32_t tf = __float_as_uint(prm.t_full) & 0x7FFFFFFFu;
  const int nq = dpad / 4;  // column quads (keys past d are never counted)
  if (prm.mode != SPAX_MASK_TOPK) {
    uint32_t c1 = 0, c2 = 0;
    for (int i = tid; i < nq; i += kMaskThreads) {
      const uint4 k4 = reinterpret_cast<const uint4*>(keys)[i];
      const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool ok = 4 * i + e < d;
        c1 += ok && kk[e] < ts;
        c2 += ok && kk[e] < tf;
      }
    }
    const uint32_t both = block_sum(c1 | (c2 << 16), s_warp, &s_total);  // d <= 32768: no carry
    n1 = both & 0xFFFFu;
    n2 = both >> 16;
  }

  // ---- TopK targets: K1 = #full, K2 = #full + #approx (largest first) ----
  uint32_t K0 = 0, K1 = 0;
  if (prm.mode == SPAX_MASK_TOPK) {
    K0 = (uint32_t)prm.k_full;
    K1 = (uint32_t)prm.k_full + (uint32_t)prm.k_approx;
  } else if (prm.mode == SPAX_MASK_GUIDED) {
    const long long m1 = guided_clip(n1, d, prm.s_skip_bp, prm.delta_bp);
    long long m2 = guided_clip(n2, d, prm.s_below_full_bp, prm.delta_bp);
    if (m2 < m1) m2 = m1;
    K0 = (uint32_t)(d - m2);
    K1 = (uint32_t)(d - m1);
  }
  const bool topk_like = prm.mode != SPAX_MASK_THRESHOLD;
  const bool act0 = topk_like && K0 > 0, act1 = topk_like && K1 > 0;

  // warp segments for the ordered passes: warp w owns columns [sw0, sw1)
  const int seg = ((d + 32 * kMaskWarps - 1) / (32 * kMaskWarps)) * 32;
  const int sw0 = min(d, wid * seg), sw1 = min(d, sw0 + seg);

  bool fast = true;
  uint32_t V0 = 0u, V1 = 0u, rem0 = 0u, rem1 = 0u;
  if (act0 || act1) {
    // ---- fast path: coarse (exponent) and fine (exponent + 7 mantissa bits) histograms ----
    for (int i = tid; i < (kFineWords + kCoarseBins) / 4; i += kMaskThreads)
      reinterpret_cast<uint4*>(fine)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    for (int i = tid; i < nq; i += kMaskThreads) {
      const uint4 k4 = reinterpret_cast<const uint4*>(keys)[i];
      const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (4 * i + e < d) {
          const uint32_t b = kk[e] >> 16;
          atomicAdd(&fine[b >> 1], 1u << ((b & 1u) << 4));
          atomicAdd(&coarse[b >> 7], 1u);
        }
      }
    }
    __syncthreads();
    if (wid < 2 && (wid ? act1 : act0)) {
      // warp k finds boundary k: coarse bin (8 per lane, from the top), then the fine bin
      // among the 128 under it (4 per lane)
      const uint32_t Kw = wid ? K1 : K0;
      int cb;
      uint32_t above_c;
      warp_find_from_top<kCoarseBins / 32>(
          Kw, 0u, [&](int i) { return coarse[kCoarseBins - 1 - i]; }, &cb, &above_c);
      const int ecb = kCoarseBins - 1 - cb;  // the coarse bin itself (an exponent)
      int fb;
      uint32_t above_f;
      warp_find_from_top<4>(
          Kw, above_c,
          [&](int i) {
            const int b = ecb * 128 + 127 - i;
            return (fine[b >> 1] >> ((b & 1) << 4)) & 0xFFFFu;
          },
          &fb, &above_f);
      if (lane == 0) {
        s_bin[wid] = (uint32_t)(ecb * 128 + 127 - fb);
        s_above[wid] = above_f;
      }
    }
    __syncthreads();
    // ---- candidates: the keys of each boundary bin ----
    uint32_t* ck = fine;                                           // [2][kCandCap] keys
    int32_t* ci = reinterpret_cast<int32_t*>(fine + 2 * kCandCap);  // [2][kCandCap] columns
    const uint32_t bin0 = act0 ? s_bin[0] : 0xFFFFFFFFu, bin1 = act1 ? s_bin[1] : 0xFFFFFFFFu;
    for (int i = tid; i < nq; i += kMaskThreads) {
      const uint4 k4 = reinterpret_cast<const uint4*>(keys)[i];
      const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * i + e;
        const uint32_t k = kk[e], b = k >> 16;
        if (j < d && b == bin0) {
          const uint32_t pos = atomicAdd(&s_cc[0], 1u);
          if (pos < kCandCap) {
            ck[pos] = k;
            ci[pos] = j;
          }
        }
        if (j < d && b == bin1) {
          const uint32_t pos = atomicAdd(&s_cc[1], 1u);
          if (pos < kCandCap) {
            ck[kCandCap + pos] = k;
            ci[kCandCap + pos] = j;
          }
        }
      }
    }
    __syncthreads();
    fast = s_cc[0] <= kCandCap && s_cc[1] <= kCandCap;
    if (fast) {
      // exact rank of each boundary key within its bin (key desc, column asc), one warp per key;
      // one target at a time so that no two threads update the same flag byte
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int c = (int)s_cc[k];
        const uint32_t* kk = ck + k * kCandCap;
        const int32_t* ii = ci + k * kCandCap;
        const uint32_t Kk = k ? K1 : K0;
        for (int i = wid; i < c; i += kMaskWarps) {
          const uint32_t key = kk[i];
          const int32_t col = ii[i];
          uint32_t r = 0;
          for (int q = lane; q < c; q += 32) r += (kk[q] > key) || (kk[q] == key && ii[q] < col);
          r = __reduce_add_sync(0xffffffffu, r);
          if (lane == 0 && s_above[k] + r < Kk) flags[col] |= (uint8_t)(1u << k);
        }
        __syncthreads();
      }
    } else {
      // ---- fallback: radix select (11/11/9 bits) of the K-th largest key for both targets ----
      uint32_t* hist = fine;  // [2][2048]
      constexpr int kBpt = 2048 / kMaskThreads;  // bins per thread in the top-down scan
      rem0 = K0;
      rem1 = K1;
#pragma unroll
      for (int pass = 0; pass < 3; ++pass) {
        const int bits = pass == 2 ? 9 : 11;
        const int sh = pass == 0 ? 20 : (pass == 1 ? 9 : 0), nb = 1 << bits, hs = sh + bits;
        for (int i = tid; i < 2 * 2048; i += kMaskThreads) hist[i] = 0;
        __syncthreads();
        for (int j = tid; j < d; j += kMaskThreads) {
          const uint32_t k = keys[j];
          if (act0 && (k >> hs) == (V0 >> hs)) atomicAdd(&hist[(k >> sh) & (nb - 1)], 1u);
          if (act1 && (k >> hs) == (V1 >> hs)) atomicAdd(&hist[2048 + ((k >> sh) & (nb - 1))], 1u);
        }
        __syncthreads();
        // warp-level scans from the top: thread i owns bins nb-1-kBpt*i ... (both targets)
        uint32_t h0[kBpt], h1[kBpt], t0 = 0, t1 = 0;
#pragma unroll
        for (int q = 0; q < kBpt; ++q) {
          const int b = nb - 1 - kBpt * tid - q;
          h0[q] = b >= 0 ? hist[b] : 0u;
          h1[q] = b >= 0 ? hist[2048 + b] : 0u;
          t0 += h0[q];
          t1 += h1[q];
        }
        const uint32_t packed = t0 | (t1 << 16);
        uint32_t incl = packed;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += n;
        }
        const uint32_t woff = warps_excl_scan(__shfl_sync(0xffffffffu, incl, 31), s_warp, &s_total);
        const uint32_t abv = woff + incl - packed;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!(t ? act1 : act0)) continue;
          const uint32_t rem = t ? rem1 : rem0;
          uint32_t cum = (abv >> (16 * t)) & 0xFFFFu;
          const uint32_t tt = t ? t1 : t0;
          if (cum < rem && rem <= cum + tt) {
#pragma unroll
            for (int q = 0; q < kBpt; ++q) {
              const uint32_t hq = t ? h1[q] : h0[q];
              if (cum < rem && rem <= cum + hq) {
                s_sel_bin[t] = (uint32_t)(nb - 1 - kBpt * tid - q);
                s_sel_rem[t] = rem - cum;
              }
              cum += hq;
            }
          }
        }
        __syncthreads();
        if (act0) {
          V0 |= s_sel_bin[0] << sh;
          rem0 = s_sel_rem[0];
        }
        if (act1) {
          V1 |= s_sel_bin[1] << sh;
          rem1 = s_sel_rem[1];
        }
        __syncthreads();
      }
      // ordered equal-key ranks: the first rem_t columns (ascending) with key == V_t are in
      uint32_t e0 = 0, e1 = 0;
      for (int b = sw0; b < sw1; b += 32) {
        const int j = b + lane;
        const uint32_t k = j < sw1 ? keys[j] : 0xFFFFFFFFu;
        e0 += __popc(__ballot_sync(0xffffffffu, k == V0));
        e1 += __popc(__ballot_sync(0xffffffffu, k == V1));
      }
      const uint32_t eoff = warps_excl_scan(e0 | (e1 << 16), s_warp, &s_total);
      uint32_t q0 = eoff & 0xFFFFu, q1 = eoff >> 16;
      const uint32_t lt = (1u << lane) - 1u;
      for (int b = sw0; b < sw1; b += 32) {
        const int j = b + lane;
        const uint32_t k = j < sw1 ? keys[j] : 0xFFFFFFFFu;
        const uint32_t b0 = __ballot_sync(0xffffffffu, k == V0);
        const uint32_t b1 = __ballot_sync(0xffffffffu, k == V1);
        if (j < sw1) {
          const bool in0 = act0 && (k > V0 || (k == V0 && q0 + __popc(b0 & lt) < rem0));
          const bool in1 = act1 && (k > V1 || (k == V1 && q1 + __popc(b1 & lt) < rem1));
          flags[j] = (uint8_t)(in0 ? 2u : (in1 ? 1u : 0u));
        }
        q0 += __popc(b0);
        q1 += __popc(b1);
      }
      __syncthreads();
    }
  }

  // ---- tier codes (the fallback path has written them already) ----
  if (!topk_like || fast) {
    const uint32_t fb0 = act0 ? s_bin[0] : 0u, fb1 = act1 ? s_bin[1] : 0u;
    for (int i = tid; i < nq; i += kMaskThreads) {
      const uint4 k4 = reinterpret_cast<const uint4*>(keys)[i];
      const uint32_t f4 = reinterpret_cast<const uint32_t*>(flags)[i];
      const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
      uint32_t out = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t k = kk[e], f = (f4 >> (8 * e)) & 0xFFu;
        uint32_t t;
        if (!topk_like) {
          t = k < ts ? 0u : (k < tf ? 1u : 2u);
        } else {
          const uint32_t b = k >> 16;
          const bool in1 = act0 && (b > fb0 || (b == fb0 && (f & 1u)));
          const bool in2 = act1 && (b > fb1 || (b == fb1 && (f & 2u)));
          t = in1 ? 2u : (in2 ? 1u : 0u);
        }
        if (4 * i + e < d) out |= t << (8 * e);
      }
      reinterpret_cast<uint32_t*>(flags)[i] = out;  // flags now hold the tier codes
    }
    __syncthreads();
  }

  // ---- ordered compaction: lane owns 4 consecutive columns, a warp 128 per step; per-warp
  // counts, warp offsets, then shuffle-scan-positioned stores ----
  const int segq = ((nq + 32 * kMaskWarps - 1) / (32 * kMaskWarps)) * 32;  // quads per warp
  const int q0w = min(nq, wid * segq), q1w = min(nq, q0w + segq);
  uint32_t cnt = 0;  // (full | approx << 16) in this warp's segment
  for (int qb = q0w; qb < q1w; qb += 32) {
    const int q = qb + lane;
    const uint32_t f4 = q < q1w ? reinterpret_cast<const uint32_t*>(flags)[q] : 0u;
    // bytes are 0, 1, 2: byte >> 1 marks full, byte & 1 marks approx
    cnt += __popc((f4 >> 1) & 0x01010101u) | (__popc(f4 & 0x01010101u) << 16);
  }
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  const uint32_t off = warps_excl_scan(cnt, s_warp, &s_total);  // no carry: d <= 32768
  const uint32_t tot = s_total;
  uint32_t base = off;  // (full | approx << 16) running offset of this warp's next step
  for (int qb = q0w; qb < q1w; qb += 32) {
    const int q = qb + lane;
    const uint32_t f4 = q < q1w ? reinterpret_cast<const uint32_t*>(flags)[q] : 0u;
    const uint32_t mine = __popc((f4 >> 1) & 0x01010101u) | (__popc(f4 & 0x01010101u) << 16);
    uint32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    uint32_t pos = base + incl - mine;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t t = (f4 >> (8 * e)) & 0xFFu;
      if (t == 2u) full_idx[pos & 0xFFFFu] = 4 * q + e;
      if (t == 1u) approx_idx[pos >> 16] = 4 * q + e;
      pos += (t == 2u) ? 1u : (t == 1u ? 0x10000u : 0u);
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if ((reinterpret_cast<uintptr_t>(tier) & 3u) == 0) {
    for (int i = tid; i < d / 4; i += kMaskThreads)
      reinterpret_cast<uint32_t*>(tier)[i] = reinterpret_cast<const uint32_t*>(flags)[i];
    for (int j = 4 * (d / 4) + tid; j < d; j += kMaskThreads) tier[j] = flags[j];
  } else {
    for (int j = tid; j < d; j += kMaskThreads) tier[j] = flags[j];
  }
  if (tid == 0) {
    counts[0] = (int32_t)(tot & 0xFFFFu);
    counts[1] = (int32_t)(tot >> 16);
    counts[2] = (int32_t)n1;
    counts[3] = (int32_t)n2;
  }
}

cudaError_t launch_mask(const float* x, int d_in, const spax_mask_params& p, uint8_t* tier,
                        int32_t* full_idx, int32_t* approx_idx, int32_t* counts, int32_t* status,
                        cudaStream_t stream) {
  const int smem = (int)mask_smem_bytes(d_in);
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(mask_kernel), smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(mask_kernel, dim3(1), dim3(kMaskThreads), (size_t)smem, stream, x, d_in, p,
                    tier, full_idx, approx_idx, counts, status);
}

}  // namespace spax
