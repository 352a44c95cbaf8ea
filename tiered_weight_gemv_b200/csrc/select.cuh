// select.cuh — the per-token tier rule inside one CTA of 512 threads: |x| keys, the threshold
// counts, the exact boundaries of the TopK / guided rules, and the ordered compaction.
//
// Sources: SpAx (arXiv 2610.02598), Abstract — skip the columns whose activations are closest to
// zero, approximate the smaller ones, read the largest in full. TopK-Guided (arXiv 2610.01763),
// Abstract and §1 — the threshold rule (TEAL) and the fixed-count TopK rule (WINA); §2.1 — the
// natural sparsity estimated from the calibrated threshold, clipped to a ±δ band around the
// target, then TopK.
//
// Rank order: larger |x| first; equal |x| by lower column index first. |x| is handled as its
// fp32 bit pattern with the sign cleared (monotone as an unsigned integer for finite values,
// and -0.0 == +0.0).
//
// A boundary t (t = 0: full | rest; t = 1: full+approx | skip) is
//   in_t(j) = key_j >= lo_t  or  (key_j == eqv_t and j is among the first rem_t such columns),
// which covers the threshold rule (lo = threshold), a TopK boundary at the K-th largest key V
// (lo = V + 1, eqv = V, rem = K - #{key > V}; lo = V when every key equal to V is in) and the
// empty set.
//
// The kernel is bound by instruction issue (a few thousand columns, one CTA), so every pass is a
// short loop over keys held in shared memory:
//   fetch    x -> shared memory with cp.async (all loads in flight at once);
//   pass 1   a 4096-bin histogram of key bits 30..19, the threshold counts (non-finite keys land
//            in the top 16 bins); x itself stays in shared memory, and every pass clears the sign
//            bit as it loads a key;
//   find     a block-wide scan from the top: each boundary's 12-bit bin and the count above it;
//   pass 2   the keys of those bins: a 1024-bin histogram of bits 18..9 and the sub-bin of rank
//            K; when rank K is the sub-bin's last key (always, when it holds one key) the sub-bin's
//            lowest key value bounds the set and nothing more is needed;
//   pass 2b  (only otherwise) a 512-bin histogram of bits 8..0 gives V and its multiplicity;
//   pass 3   per-thread counts over a contiguous run of columns, one block scan;
//   pass 4   tier codes and the ascending lists (staged in shared memory, then copied out with
//            16-byte stores), written from the same runs.
// With a TopK guess of the two boundary keys (select_topk_guessed), one windowed pass and a
// 2048-bin scan per boundary take the place of passes 1 to 2b whenever the guess holds.
#pragma once

#include <cstddef>

#include "common.cuh"

namespace spax {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelBins = 4096;            // key bits 30..19
constexpr uint32_t kNoKey = 0xFFFFFFFFu;  // equal to no finite key
constexpr uint32_t kNoLo = 0x80000000u;   // above every finite key
constexpr int kSelCand = 32;              // keys of one window bin a guessed boundary ranks
constexpr int kGuessBins = 2048;          // bins of one guessed window (two windows fill hist)
static_assert(2 * kGuessBins <= kSelBins && kGuessBins == 1 << 11, "window bins");

struct Boundary {
  uint32_t lo, eqv, rem;
};

struct alignas(16) SelectSmem {
  uint32_t hist[kSelBins];
  uint32_t ha[2][1024];  // bits 18..9 under each boundary's 12-bit prefix
  uint32_t hb[2][512];   // bits 8..0 under a 22-bit prefix (when pass 2 leaves V open)
  uint32_t stat[4];      // #keys < t_skip, #keys < t_full, non-finite flag
  uint32_t sel[2][4];    // per boundary: prefix / key, count above, count in the bin
  alignas(16) uint32_t wsum[kSelWarps];
  alignas(16) uint32_t wscan[kSelWarps];
  uint32_t hint[8];           // guessed TopK: #keys above each window (0, 2), the largest key
                              // (4), the keys gathered from one bin per boundary (5, 6)
  uint32_t cand[2][kSelCand]; // guessed TopK: those gathered keys
};

// Dynamic shared memory the keys of d columns take (padded to whole 16-byte quads).
__host__ __device__ inline size_t select_keys_bytes(int d) { return (size_t(d) + 3) / 4 * 16; }
// Dynamic shared memory of the staged lists: d 16-bit column indices, the approximate list
// starting 8-byte aligned, and room for the 4-entry reads that copy them out.
__host__ __device__ inline size_t select_list_bytes(int d) { return (2 * (size_t(d) + 16) + 15) / 16 * 16; }

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

// Zero what the selection accumulates into (all threads; may run before the wait on the
// preceding kernel). hist, ha and hb are one run of words, cleared with 16-byte stores.
__device__ __forceinline__ void select_zero(SelectSmem& S) {
  constexpr int kZeroQuads = (kSelBins + 2 * 1024 + 2 * 512) / 4;
  static_assert(offsetof(SelectSmem, ha) == kSelBins * 4 &&
                    offsetof(SelectSmem, hb) == (kSelBins + 2 * 1024) * 4 && kSelBins % 4 == 0,
                "hist, ha and hb must be one run of 16-byte quads");
  uint4* z = reinterpret_cast<uint4*>(S.hist);
#pragma unroll
  for (int k = 0; k < (kZeroQuads + kSelThreads - 1) / kSelThreads; ++k) {
    const int i = (int)threadIdx.x + k * kSelThreads;
    if (i < kZeroQuads) z[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (threadIdx.x < 4) S.stat[threadIdx.x] = 0u;
  if (threadIdx.x < 8) S.hint[threadIdx.x] = 0u;
}

// x[0, d) -> keys[] as raw fp32 bits; the tail of the last quad is zero. Ends with a barrier.
__device__ __forceinline__ void select_fetch(const float* __restrict__ x, int d,
                                             uint32_t* __restrict__ keys) {
  const int tid = threadIdx.x;
  const int nfull = d >> 2;  // quads fully inside x
  if ((reinterpret_cast<uintptr_t>(x) & 15u) == 0) {
    for (int q = tid; q < nfull; q += kSelThreads)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(keys + 4 * q)),
                   "l"(x + 4 * q)
                   : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
  } else {
    for (int j = tid; j < 4 * nfull; j += kSelThreads) keys[j] = __float_as_uint(__ldg(x + j));
  }
  if (tid < 4 && (d & 3)) {
    const int j = 4 * nfull + tid;
    keys[j] = j < d ? __float_as_uint(__ldg(x + j)) : 0u;
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
}

// x_j = swiglu_x(g_j, u_j) from gu = [g; u] (2 d values) -> keys[] as raw fp32 bits, the tail
// of the last quad zero; x_out (may be null) receives x. Ends with a barrier.
// Out of line (as is select_fetch_scored): only the chained-layer entry point runs it, and code
// inlined into the hot path costs instruction fetch even where it never executes.
static __device__ __noinline__ void select_fetch_swiglu(const float* __restrict__ gu, int d,
                                                    uint32_t* __restrict__ keys,
                                                    float* __restrict__ x_out) {
  const int tid = threadIdx.x;
  const float* g = gu;
  const float* u = gu + d;
  const bool vec = ((reinterpret_cast<uintptr_t>(g) | reinterpret_cast<uintptr_t>(u) |
                     reinterpret_cast<uintptr_t>(x_out)) & 15u) == 0;
  const int nfull = d >> 2;
  if (vec) {  // batches of kB quads per thread: all loads of a batch in flight together
    constexpr int kB = 6;
    for (int q0 = tid; q0 < nfull; q0 += kB * kSelThreads) {
      float4 a[kB], b[kB];
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int q = q0 + k * kSelThreads;
        if (q < nfull) {
          a[k] = __ldg(reinterpret_cast<const float4*>(g) + q);
          b[k] = __ldg(reinterpret_cast<const float4*>(u) + q);
        }
      }
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int q = q0 + k * kSelThreads;
        if (q < nfull) {
          const float4 v = make_float4(swiglu_x(a[k].x, b[k].x), swiglu_x(a[k].y, b[k].y),
                                       swiglu_x(a[k].z, b[k].z), swiglu_x(a[k].w, b[k].w));
          reinterpret_cast<float4*>(keys)[q] = v;
          if (x_out) reinterpret_cast<float4*>(x_out)[q] = v;
        }
      }
    }
  } else {
    for (int j = tid; j < 4 * nfull; j += kSelThreads) {
      const float v = swiglu_x(__ldg(g + j), __ldg(u + j));
      keys[j] = __float_as_uint(v);
      if (x_out) x_out[j] = v;
    }
  }
  if (tid < 4 && (d & 3)) {
    const int j = 4 * nfull + tid;
    float v = 0.f;
    if (j < d) {
      v = swiglu_x(__ldg(g + j), __ldg(u + j));
      if (x_out) x_out[j] = v;
    }
    keys[j] = j < d ? __float_as_uint(v) : 0u;
  }
  __syncthreads();
}

// WINA score keys: keys[j] = bits(|x_j| * norm_j) (one correctly rounded fp32 product; x and
// the norms read in batches ahead of the arithmetic), the tail of the last quad zero. Ends with
// a barrier.
static __device__ __noinline__ void select_fetch_scored(const float* __restrict__ x,
                                                    const float* __restrict__ norms, int d,
                                                    uint32_t* __restrict__ keys) {
  const int tid = threadIdx.x;
  const int nfull = d >> 2;
  auto score = [](float a, float n) { return __float_as_uint(__fmul_rn(fabsf(a), n)); };
  if (((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(norms)) & 15u) == 0) {
    constexpr int kB = 6;
    for (int q0 = tid; q0 < nfull; q0 += kB * kSelThreads) {
      float4 a[kB], n[kB];
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int q = q0 + k * kSelThreads;
        if (q < nfull) {
          a[k] = __ldg(reinterpret_cast<const float4*>(x) + q);
          n[k] = __ldg(reinterpret_cast<const float4*>(norms) + q);
        }
      }
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int q = q0 + k * kSelThreads;
        if (q < nfull)
          reinterpret_cast<uint4*>(keys)[q] = make_uint4(score(a[k].x, n[k].x), score(a[k].y, n[k].y),
                                                         score(a[k].z, n[k].z), score(a[k].w, n[k].w));
      }
    }
  } else {
    for (int j = tid; j < 4 * nfull; j += kSelThreads) keys[j] = score(__ldg(x + j), __ldg(norms + j));
  }
  if (tid < 4 && (d & 3)) {
    const int j = 4 * nfull + tid;
    keys[j] = j < d ? score(__ldg(x + j), __ldg(norms + j)) : 0u;
  }
  __syncthreads();
}

// The |x| keys of quad q: x is kept as it is in shared memory (the product reads its signs back
// from there), so every pass clears the sign bits as it loads.
__device__ __forceinline__ uint4 ld_key4(const uint4* kq, int q) {
  uint4 v = kq[q];
  v.x &= 0x7FFFFFFFu, v.y &= 0x7FFFFFFFu, v.z &= 0x7FFFFFFFu, v.w &= 0x7FFFFFFFu;
  return v;
}

// Pass 1: the threshold counts, the non-finite flag and (mode != 0) the 12-bit histogram of the
// |x| keys (x itself stays in keys[]). mode: 0 threshold, 1 TopK, 2 guided. Ends with a barrier;
// n1, n2 and bad are identical in every thread.
__device__ __forceinline__ void select_pass1(int mode, int d, uint32_t ts, uint32_t tf,
                                             const uint32_t* __restrict__ keys, SelectSmem& S,
                                             uint32_t* n1, uint32_t* n2, bool* bad) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int nq = (d + 3) >> 2;
  const uint4* kq = reinterpret_cast<const uint4*>(keys);
  uint32_t cs = 0, cf = 0, b = 0;
  if (mode == SPAX_MASK_TOPK) {
    for (int q = tid; q < nq; q += kSelThreads) {
      const uint4 v = ld_key4(kq, q);
      atomicAdd(&S.hist[v.x >> 19], 1u);
      atomicAdd(&S.hist[v.y >> 19], 1u);
      atomicAdd(&S.hist[v.z >> 19], 1u);
      atomicAdd(&S.hist[v.w >> 19], 1u);
    }
  } else {
    const bool hist = mode == SPAX_MASK_GUIDED;
    for (int q = tid; q < nq; q += kSelThreads) {
      const uint4 v = ld_key4(kq, q);
      cs += (v.x < ts) + (v.y < ts) + (v.z < ts) + (v.w < ts);
      cf += (v.x < tf) + (v.y < tf) + (v.z < tf) + (v.w < tf);
      b = max(b, max(max(v.x, v.y), max(v.z, v.w)));
      if (hist) {
        atomicAdd(&S.hist[v.x >> 19], 1u);
        atomicAdd(&S.hist[v.y >> 19], 1u);
        atomicAdd(&S.hist[v.z >> 19], 1u);
        atomicAdd(&S.hist[v.w >> 19], 1u);
      }
    }
    b = b >= 0x7F800000u;
  }
  // the zero keys padding the last quad are not columns
  const uint32_t pad = (uint32_t)(4 * nq - d);
  if (tid == 0 && pad) {
    if (mode != SPAX_MASK_THRESHOLD) atomicSub(&S.hist[0], pad);
    cs -= ts > 0u ? pad : 0u;
    cf -= tf > 0u ? pad : 0u;
  }
  if (mode != SPAX_MASK_TOPK) {
    cs = __reduce_add_sync(0xffffffffu, cs);
    cf = __reduce_add_sync(0xffffffffu, cf);
    b = __reduce_or_sync(0xffffffffu, b);
    if (lane == 0) {
      if (cs) atomicAdd(&S.stat[0], cs);
      if (cf) atomicAdd(&S.stat[1], cf);
      if (b) S.stat[2] = 1u;
    }
  }
  __syncthreads();
  *n1 = S.stat[0];
  *n2 = S.stat[1];
  if (mode == SPAX_MASK_THRESHOLD) {
    *bad = S.stat[2] != 0u;
  } else {  // key bits 30..19 >= 0xFF0 <=> exponent all ones (Inf / NaN)
    const uint4 a = *reinterpret_cast<const uint4*>(&S.hist[kSelBins - 16 + 4 * (lane & 3)]);
    const bool nz = (a.x | a.y | a.z | a.w) != 0u;
    *bad = __any_sync(0xffffffffu, nz && lane < 4);
  }
}

// c[i] = h[top - i] for i < PER (top - PER + 1 a multiple of 4: vector loads).
template <int PER>
__device__ __forceinline__ void load_desc(const uint32_t* h, int top, uint32_t (&c)[PER]) {
  if constexpr (PER % 4 == 0) {
#pragma unroll
    for (int g = 0; g < PER / 4; ++g) {
      const uint4 q = *reinterpret_cast<const uint4*>(h + top - 4 * g - 3);
      c[4 * g] = q.w, c[4 * g + 1] = q.z, c[4 * g + 2] = q.y, c[4 * g + 3] = q.x;
    }
  } else {
    static_assert(PER == 2, "2 or a multiple of 4 entries per thread");
    const uint2 q = *reinterpret_cast<const uint2*>(h + top - 1);
    c[0] = q.y, c[1] = q.x;
  }
}

// Both boundaries at once: threads [0, 256) search h0 for rank K0, threads [256, 512) search h1
// for K1 (counts above the histograms ab0 / ab1); each thread owns NB / 256 consecutive bins from
// the top. Writes S.sel[t] = {pre_t << bits | bin, count above the bin, count in the bin}.
// Ends with a barrier.
template <int NB>
__device__ __forceinline__ void block_find_pair(const uint32_t* h0, const uint32_t* h1, bool act0,
                                                bool act1, uint32_t K0, uint32_t K1, uint32_t ab0,
                                                uint32_t ab1, uint32_t pre0, uint32_t pre1,
                                                int bits, SelectSmem& S) {
  constexpr int PER = NB / 256;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int t = tid >> 8, u = tid & 255;
  uint32_t c[PER], s = 0;
  load_desc<PER>(t ? h1 : h0, NB - 1 - PER * u, c);
#pragma unroll
  for (int i = 0; i < PER; ++i) s += c[i];
  uint32_t incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) S.wsum[wid] = incl;
  __syncthreads();
  uint32_t cum = (t ? ab1 : ab0) + incl - s;
  {  // counts of the warps before this one in its half (8 per half), as two vector loads
    const uint4 lo = *reinterpret_cast<const uint4*>(&S.wsum[8 * t]);
    const uint4 hi = *reinterpret_cast<const uint4*>(&S.wsum[8 * t + 4]);
    const uint32_t w8[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    const int wl = wid - 8 * t;
#pragma unroll
    for (int w = 0; w < 8; ++w) cum += w < wl ? w8[w] : 0u;
  }
  const uint32_t K = t ? K1 : K0;
  if ((t ? act1 : act0) && cum < K && K <= cum + s) {
    uint32_t a = cum;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      if (a < K && K <= a + c[i]) {
        S.sel[t][0] = ((t ? pre1 : pre0) << bits) | (uint32_t)(NB - 1 - (PER * u + i));
        S.sel[t][1] = a;
        S.sel[t][2] = c[i];
      }
      a += c[i];
    }
  }
  __syncthreads();
}

// The two boundaries of the rule (after select_pass1; all threads; barriers inside). B is
// identical in every thread.
__device__ __forceinline__ void select_boundaries(const spax_mask_params& prm, int d,
                                                  const uint32_t* __restrict__ keys, uint32_t n1,
                                                  uint32_t n2, SelectSmem& S, Boundary* B) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nq = (d + 3) >> 2;
  const uint32_t pad = (uint32_t)(4 * nq - d);
  const uint4* kq = reinterpret_cast<const uint4*>(keys);
  const uint32_t ts = __float_as_uint(prm.t_skip) & 0x7FFFFFFFu;
  const uint32_t tf = __float_as_uint(prm.t_full) & 0x7FFFFFFFu;
  // K0 = #full, K1 = #full + #approx; kind 0 = empty, 1 = threshold, 2 = TopK selection
  uint32_t K0 = 0, K1 = 0;
  int kind0 = 1, kind1 = 1;
  if (prm.mode == SPAX_MASK_TOPK) {
    K0 = (uint32_t)prm.k_full;
    K1 = (uint32_t)prm.k_full + (uint32_t)prm.k_approx;
    kind0 = K0 ? 2 : 0;
    kind1 = K1 ? 2 : 0;
  } else if (prm.mode == SPAX_MASK_GUIDED) {
    const long long m1 = guided_clip(n1, d, prm.s_skip_bp, prm.delta_bp);
    long long m2 = guided_clip(n2, d, prm.s_below_full_bp, prm.delta_bp);
    if (m2 < m1) m2 = m1;
    K0 = (uint32_t)(d - m2);
    K1 = (uint32_t)(d - m1);
    // a count equal to the threshold count selects exactly the threshold set
    kind0 = K0 == (uint32_t)d - n2 ? 1 : (K0 ? 2 : 0);
    kind1 = K1 == (uint32_t)d - n1 ? 1 : (K1 ? 2 : 0);
  }
  const bool sel0 = kind0 == 2, sel1 = kind1 == 2;
  uint32_t V0 = 0, V1 = 0, ab0 = 0, ab1 = 0, cnt0 = 0, cnt1 = 0;  // key, #above, #equal
  if (sel0 || sel1) {
    // ---- find: 12-bit bins; thread t owns bins 4095-8t .. 4088-8t (high to low) ----
    {
      constexpr int PER = kSelBins / kSelThreads;
      uint32_t c[PER], s = 0;
      load_desc<PER>(S.hist, kSelBins - 1 - PER * tid, c);
#pragma unroll
      for (int i = 0; i < PER; ++i) s += c[i];
      uint32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      if (lane == 31) S.wsum[wid] = incl;
      __syncthreads();
      uint32_t cum = incl - s;
#pragma unroll
      for (int g = 0; g < kSelWarps / 4; ++g) {  // counts of the warps before this one
        const uint4 q = *reinterpret_cast<const uint4*>(&S.wsum[4 * g]);
        cum += (4 * g + 0 < wid ? q.x : 0u) + (4 * g + 1 < wid ? q.y : 0u) +
               (4 * g + 2 < wid ? q.z : 0u) + (4 * g + 3 < wid ? q.w : 0u);
      }
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const uint32_t K = t ? K1 : K0;
        if ((t ? sel1 : sel0) && cum < K && K <= cum + s) {
          uint32_t a = cum;
#pragma unroll
          for (int i = 0; i < PER; ++i) {
            if (a < K && K <= a + c[i]) {
              S.sel[t][0] = (uint32_t)(kSelBins - 1 - (PER * tid + i));
              S.sel[t][1] = a;
            }
            a += c[i];
          }
        }
      }
      __syncthreads();
    }
    const uint32_t p0 = sel0 ? S.sel[0][0] : kNoKey, p1 = sel1 ? S.sel[1][0] : kNoKey;
    ab0 = sel0 ? S.sel[0][1] : 0u;
    ab1 = sel1 ? S.sel[1][1] : 0u;
    // ---- pass 2: bits 18..9 of the keys in the two bins. One atomic per key of either bin
    // (both boundaries in one bin share ha[0]); a warp whose keys all miss skips the atomics.
    const bool same = p0 == p1;
    for (int qb = tid - lane; qb < nq; qb += kSelThreads) {  // warp-uniform trip count
      const int q = qb + lane;
      const uint4 v = q < nq ? ld_key4(kq, q) : make_uint4(kNoKey, kNoKey, kNoKey, kNoKey);
      const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t b = kk[e] >> 19;
        const bool m = b == p0 || b == p1;
        if (__any_sync(0xffffffffu, m) && m)
          atomicAdd(&S.ha[b == p0 ? 0 : 1][(kk[e] >> 9) & 1023u], 1u);
      }
    }
    if (tid == 0 && pad) {  // padding zeros of the last quad
      if (p0 == 0u) atomicSub(&S.ha[0][0], pad);
      else if (p1 == 0u) atomicSub(&S.ha[1][0], pad);
    }
    __syncthreads();
    block_find_pair<1024>(S.ha[0], same ? S.ha[0] : S.ha[1], sel0, sel1, K0, K1, ab0, ab1, p0, p1,
                          10, S);
    // resolved here when rank K is the sub-bin's last key: then the whole sub-bin is in
    bool need0 = false, need1 = false;
    uint32_t q0 = kNoKey, q1 = kNoKey;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (!(t ? sel1 : sel0)) continue;
      const uint32_t pre = S.sel[t][0], above = S.sel[t][1], c = S.sel[t][2];
      const uint32_t rem = (t ? K1 : K0) - above;
      uint32_t V, ab, cnt;
      bool need = false;
      if (rem == c) {  // all of the sub-bin: its smallest key bounds the set from below
        V = pre << 9;
        ab = above;
        cnt = kNoKey;  // marks "every key >= V is in"
      } else {
        need = true;
        V = 0, ab = 0, cnt = 0;
      }
      if (t) {
        V1 = V, ab1 = ab, cnt1 = cnt, need1 = need, q1 = need ? pre : kNoKey;
      } else {
        V0 = V, ab0 = ab, cnt0 = cnt, need0 = need, q0 = need ? pre : kNoKey;
      }
    }
    // ---- pass 2b: bits 8..0 under the 22-bit prefix ----
    if (need0 || need1) {
      const uint32_t abA0 = S.sel[0][1], abA1 = S.sel[1][1];
      __syncthreads();  // S.sel is rewritten below
      const bool same2 = q0 == q1;
      for (int qb = tid - lane; qb < nq; qb += kSelThreads) {  // warp-uniform trip count
        const int q = qb + lane;
        const uint4 v = q < nq ? ld_key4(kq, q) : make_uint4(kNoKey, kNoKey, kNoKey, kNoKey);
        const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t b = kk[e] >> 9;
          const bool m = b == q0 || b == q1;
          if (__any_sync(0xffffffffu, m) && m) atomicAdd(&S.hb[b == q0 ? 0 : 1][kk[e] & 511u], 1u);
        }
      }
      if (tid == 0 && pad) {
        if (q0 == 0u) atomicSub(&S.hb[0][0], pad);
        else if (q1 == 0u) atomicSub(&S.hb[1][0], pad);
      }
      __syncthreads();
      block_find_pair<512>(S.hb[0], same2 ? S.hb[0] : S.hb[1], need0, need1, K0, K1, abA0, abA1, q0,
                           q1, 9, S);
      if (need0) V0 = S.sel[0][0], ab0 = S.sel[0][1], cnt0 = S.sel[0][2];
      if (need1) V1 = S.sel[1][0], ab1 = S.sel[1][1], cnt1 = S.sel[1][2];
    }
  }
  // ---- boundary descriptions ----
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int kind = t ? kind1 : kind0;
    if (kind == 2) {
      const uint32_t V = t ? V1 : V0, rem = (t ? K1 : K0) - (t ? ab1 : ab0);
      const uint32_t cnt = t ? cnt1 : cnt0;  // keys equal to V (0: unknown; kNoKey: all in)
      if (cnt == kNoKey || rem == cnt) {
        B[t].lo = V;
        B[t].eqv = kNoKey;
        B[t].rem = 0u;
      } else {
        B[t].lo = V + 1u;
        B[t].eqv = V;
        B[t].rem = rem;
      }
    } else if (kind == 1) {
      B[t].lo = t ? ts : tf;
      B[t].eqv = kNoKey;
      B[t].rem = 0u;
    } else {
      B[t].lo = kNoLo;
      B[t].eqv = kNoKey;
      B[t].rem = 0u;
    }
  }
}

// The window of a guess h of a boundary key: keys [lo, lo + (kGuessBins << sh)), lo the key of
// 7h/8 and the span reaching at least to the key of 9h/8 (at most 2^23 keys: the two values are
// less than a factor 2 apart). False when h is not a positive finite number or 7h/8 rounds to
// zero.
__device__ __forceinline__ bool guess_window(float h, uint32_t* lo, int* sh) {
  if (__float_as_uint(h) - 1u >= 0x7F7FFFFFu) return false;  // NaN, Inf, negative or zero
  const uint32_t a = __float_as_uint(h * 0.875f), b = __float_as_uint(h * 1.125f);
  if (a == 0u) return false;
  const uint32_t r = b - a;
  *lo = a;
  *sh = r <= (uint32_t)kGuessBins ? 0 : 32 - __clz((r - 1u) >> 11);
  return true;
}

// TopK boundaries found from a guess of each boundary key: the calibrated thresholds a caller may
// pass in t_full (boundary 0) and t_skip (boundary 1), which the TopK rule has no other use for.
// One pass over the keys counts, per boundary, the keys above a window around its guess and
// histograms the keys inside it (kGuessBins bins of 2^sh keys each, the two windows side by side
// in S.hist). When each rank K lies inside its window, a block scan of the histograms gives the
// bin of rank K; where that bin also holds keys ranked after K its keys are gathered and ranked
// among themselves. Returns 1 when B is set, 2 on a non-finite key (B unset), 0 when the guesses
// do not apply or miss, or a bin is too crowded to rank (S.hist is zero again then: the unhinted
// selection follows). The guess decides only how the boundaries are found: B describes the same
// two sets either way. All threads; barriers inside.
__device__ __forceinline__ int select_topk_guessed(const spax_mask_params& prm, int d,
                                                   const uint32_t* __restrict__ keys,
                                                   SelectSmem& S, Boundary* B) {
  const uint32_t K0 = (uint32_t)prm.k_full, K1 = (uint32_t)prm.k_full + (uint32_t)prm.k_approx;
  const bool act0 = K0 > 0u && K0 < (uint32_t)d, act1 = K1 > 0u && K1 < (uint32_t)d;
  uint32_t lo0 = 0u, lo1 = 0u;
  int sh0 = 0, sh1 = 0;
  if (!act0 && !act1) return 0;
  if (act0 && !guess_window(prm.t_full, &lo0, &sh0)) return 0;
  if (act1 && !guess_window(prm.t_skip, &lo1, &sh1)) return 0;
  const int tid = threadIdx.x, lane = tid & 31;
  const int nq = (d + 3) >> 2;
  const uint4* kq = reinterpret_cast<const uint4*>(keys);
  // ---- one pass: keys above each window, the window histograms, the largest key. The zero
  // keys padding the last quad lie below every window (lo >= 1) and count nowhere. ----
  const uint32_t w0 = act0 ? ((uint32_t)kGuessBins << sh0) : 0u;
  const uint32_t w1 = act1 ? ((uint32_t)kGuessBins << sh1) : 0u;
  uint32_t* h0 = S.hist;
  uint32_t* h1 = S.hist + kGuessBins;
  const uint32_t hi0 = lo0 + w0, hi1 = lo1 + w1;
  if (tid < 2) S.sel[tid][0] = kNoKey;  // stays when rank K is outside the window (a miss)
  uint32_t a0 = 0, a1 = 0, mx = 0;
  // disjoint windows (the usual case): one atomic per key, into whichever window holds it
  const bool disjoint = hi0 <= lo1 || hi1 <= lo0;
  for (int q = tid; q < nq; q += kSelThreads) {
    const uint4 v = ld_key4(kq, q);
    const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t k = kk[e], r0 = k - lo0, r1 = k - lo1;
      mx = max(mx, k);
      a0 += k >= hi0;
      a1 += k >= hi1;
      const bool in0 = r0 < w0, in1 = r1 < w1;
      if (disjoint) {
        if (in0 || in1) atomicAdd(in0 ? &h0[r0 >> sh0] : &h1[r1 >> sh1], 1u);
      } else {
        if (in0) atomicAdd(&h0[r0 >> sh0], 1u);
        if (in1) atomicAdd(&h1[r1 >> sh1], 1u);
      }
    }
  }
  a0 = __reduce_add_sync(0xffffffffu, a0);
  a1 = __reduce_add_sync(0xffffffffu, a1);
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (lane == 0) {
    atomicAdd(&S.hint[0], a0);
    atomicAdd(&S.hint[2], a1);
    atomicMax(&S.hint[4], mx);
  }
  __syncthreads();
  if (S.hint[4] >= 0x7F800000u) return 2;  // Inf / NaN among the keys
  const uint32_t A0 = S.hint[0], A1 = S.hint[2];
  auto unwind = [&]() {  // a miss (block-uniform): the unhinted selection needs S.hist zero
    for (int i = 4 * tid; i < kSelBins; i += 4 * kSelThreads)
      *reinterpret_cast<uint4*>(&S.hist[i]) = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();  // pass 1 adds into S.hist at once: every bin is zero before any thread does
    return 0;
  };
  // rank K lies in the window iff the scan from the top finds it before the window's bottom
  block_find_pair<kGuessBins>(h0, h1, act0, act1, K0, K1, A0, A1, 0u, 0u, 0, S);
  if (__builtin_expect((act0 && S.sel[0][0] == kNoKey) || (act1 && S.sel[1][0] == kNoKey), 0))
    return unwind();
  // ---- per boundary: the bin of rank K, the count above it and in it ----
  uint32_t base[2], above[2], cnt[2];
  bool need[2];
  bool crowded = false;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const uint32_t K = t ? K1 : K0;
    need[t] = false;
    base[t] = above[t] = cnt[t] = 0u;
    if (!(t ? act1 : act0)) {
      B[t].lo = K ? 0u : kNoLo;  // K = d: every column; K = 0: none
      B[t].eqv = kNoKey;
      B[t].rem = 0u;
      continue;
    }
    const int sh = t ? sh1 : sh0;
    base[t] = (t ? lo1 : lo0) + (S.sel[t][0] << sh);
    above[t] = S.sel[t][1];
    cnt[t] = S.sel[t][2];
    const uint32_t rem = K - above[t];
    if (rem == cnt[t]) {  // the whole bin is in: its lower edge bounds the set
      B[t].lo = base[t];
      B[t].eqv = kNoKey;
      B[t].rem = 0u;
    } else if (sh == 0) {  // a one-key bin: that key, and rem of its cnt copies
      B[t].lo = base[t] + 1u;
      B[t].eqv = base[t];
      B[t].rem = rem;
    } else {
      need[t] = true;
      crowded |= cnt[t] > (uint32_t)kSelCand;
    }
  }
  if (!need[0] && !need[1]) return 1;
  if (__builtin_expect(crowded, 0)) return unwind();
  // ---- gather the keys of each unresolved bin, then rank them (one warp per boundary) ----
  const uint32_t g0 = base[0], g1 = base[1];
  const uint32_t gw0 = need[0] ? (1u << sh0) : 0u, gw1 = need[1] ? (1u << sh1) : 0u;
  for (int q = tid; q < nq; q += kSelThreads) {
    const uint4 v = ld_key4(kq, q);
    const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (kk[e] - g0 < gw0) {
        const uint32_t i = atomicAdd(&S.hint[5], 1u);
        if (i < (uint32_t)kSelCand) S.cand[0][i] = kk[e];
      }
      if (kk[e] - g1 < gw1) {
        const uint32_t i = atomicAdd(&S.hint[6], 1u);
        if (i < (uint32_t)kSelCand) S.cand[1][i] = kk[e];
      }
    }
  }
  __syncthreads();
  // the gathered counts equal the histogram's by construction; anything else is not trusted
  if (__builtin_expect((need[0] && S.hint[5] != cnt[0]) || (need[1] && S.hint[6] != cnt[1]), 0))
    return unwind();
  const int wid = tid >> 5;
  if (wid < 2 && (wid ? need[1] : need[0])) {  // warp t ranks boundary t's keys: V, gt < rem <= gt + eq
    const uint32_t c = wid ? cnt[1] : cnt[0], ab = wid ? above[1] : above[0];
    const uint32_t rem = (wid ? K1 : K0) - ab;
    const uint32_t v = (uint32_t)lane < c ? S.cand[wid][lane] : kNoKey;
    uint32_t gt = 0, eq = 0;
    for (uint32_t j = 0; j < c; ++j) {
      const uint32_t u = __shfl_sync(0xffffffffu, v, (int)j);
      gt += u > v;
      eq += u == v;
    }
    // S.sel was read into registers before the barrier above
    if ((uint32_t)lane < c && gt < rem && rem <= gt + eq) {
      S.sel[wid][0] = v;
      S.sel[wid][1] = ab + gt;
      S.sel[wid][2] = eq;
    }
  }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (!need[t]) continue;
    const uint32_t V = S.sel[t][0], rem = (t ? K1 : K0) - S.sel[t][1], eq = S.sel[t][2];
    if (rem == eq) {
      B[t].lo = V;
      B[t].eqv = kNoKey;
      B[t].rem = 0u;
    } else {
      B[t].lo = V + 1u;
      B[t].eqv = V;
      B[t].rem = rem;
    }
  }
  return 1;
}

// x[0, d) -> keys[] as select_fetch does, through registers, summing |x| on the way: returns the
// mean |x| over the d columns (fp32, a fixed order). Ends with a barrier; S.wsum holds the warp
// sums until the rule's first scan.
__device__ __forceinline__ float select_fetch_mean(const float* __restrict__ x, int d,
                                                   uint32_t* __restrict__ keys, SelectSmem& S) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nfull = d >> 2;
  float sum = 0.f;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) == 0) {
    for (int q = tid; q < nfull; q += kSelThreads) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(x) + q);
      reinterpret_cast<float4*>(keys)[q] = v;
      sum += (fabsf(v.x) + fabsf(v.y)) + (fabsf(v.z) + fabsf(v.w));
    }
  } else {
    for (int j = tid; j < 4 * nfull; j += kSelThreads) {
      const float v = __ldg(x + j);
      keys[j] = __float_as_uint(v);
      sum += fabsf(v);
    }
  }
  if (tid < 4 && (d & 3)) {
    const int j = 4 * nfull + tid;
    const float v = j < d ? __ldg(x + j) : 0.f;
    keys[j] = __float_as_uint(v);
    sum += fabsf(v);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) S.wsum[wid] = __float_as_uint(sum);
  __syncthreads();
  float total = 0.f;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) total += __uint_as_float(S.wsum[w]);
  return total / (float)d;
}

// The TOPK_SCALED parameters as TOPK ones, given the token's mean key.
__device__ __forceinline__ spax_mask_params scaled_topk_params(const spax_mask_params& prm,
                                                               float mean) {
  spax_mask_params q = prm;
  q.mode = SPAX_MASK_TOPK;
  q.t_full = prm.t_full * mean;
  q.t_skip = prm.t_skip * mean;
  return q;
}

// TOPK_SCALED -> TOPK: the guesses t_full and t_skip, given as multiples of the token's mean key
// (mean |key| over the d columns), become keys (after a select_fetch*; all threads; one barrier).
// A non-finite or zero mean leaves no usable guess, and the TopK search then runs unhinted (which
// reports a non-finite key as the plain rule does).
__device__ __forceinline__ spax_mask_params select_scaled_topk(const spax_mask_params& prm, int d,
                                                              const uint32_t* __restrict__ keys,
                                                              SelectSmem& S) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nq = (d + 3) >> 2;
  const uint4* kq = reinterpret_cast<const uint4*>(keys);
  float sum = 0.f;  // the zero keys padding the last quad add nothing
  for (int q = tid; q < nq; q += kSelThreads) {
    const uint4 v = ld_key4(kq, q);
    sum += (__uint_as_float(v.x) + __uint_as_float(v.y)) + (__uint_as_float(v.z) + __uint_as_float(v.w));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) S.wsum[wid] = __float_as_uint(sum);  // free until the rule's first scan
  __syncthreads();
  float total = 0.f;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) total += __uint_as_float(S.wsum[w]);
  const float mean = total / (float)d;
  spax_mask_params q = prm;
  q.mode = SPAX_MASK_TOPK;
  q.t_full = prm.t_full * mean;
  q.t_skip = prm.t_skip * mean;
  return q;
}

// The rule's two boundaries (after a select_fetch*; all threads; barriers inside): the guessed
// TopK search when it applies and resolves, else pass 1 and select_boundaries. Returns true on a
// non-finite key (B unset). n1, n2: the threshold counts (0 in TopK mode).
__device__ __forceinline__ bool select_rule(const spax_mask_params& prm, int d,
                                            const uint32_t* __restrict__ keys, SelectSmem& S,
                                            uint32_t* n1, uint32_t* n2, Boundary* B) {
  if (prm.mode == SPAX_MASK_TOPK) {
    const int g = select_topk_guessed(prm, d, keys, S, B);
    if (__builtin_expect(g != 0, 1)) {
      *n1 = *n2 = 0u;
      return g == 2;
    }
  }
  const uint32_t ts = __float_as_uint(prm.t_skip) & 0x7FFFFFFFu;
  const uint32_t tf = __float_as_uint(prm.t_full) & 0x7FFFFFFFu;
  bool bad;
  select_pass1(prm.mode, d, ts, tf, keys, S, n1, n2, &bad);
  if (bad) return true;
  select_boundaries(prm, d, keys, *n1, *n2, S, B);
  return false;
}

// Exclusive block-wide prefix of one packed value per thread (two 16-bit fields, totals below
// 65536), in thread order. Returns the prefix; *total gets the sum. Two barriers (one with
// kReuse = false, when nothing writes S.wscan again before the caller's next barrier).
template <bool kReuse = true>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, SelectSmem& S, uint32_t* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) S.wscan[wid] = incl;
  __syncthreads();
  // the warp totals, one per lane, by a second shuffle scan; this warp's base from lane wid - 1
  uint32_t t = lane < kSelWarps ? S.wscan[lane] : 0u;
#pragma unroll
  for (int o = 1; o < kSelWarps; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, t, o);
    if (lane >= o) t += n;
  }
  const uint32_t base = wid ? __shfl_sync(0xffffffffu, t, wid - 1) : 0u;
  const uint32_t all = __shfl_sync(0xffffffffu, t, kSelWarps - 1);
  if (kReuse) __syncthreads();  // S.wscan may be reused right after
  *total = all;
  return base + incl - v;
}

// Ordered compaction (after select_boundaries; all threads; barriers inside). Writes the tier
// code of every column to tier[] (2 full, 1 approx, 0 skip; skipped when tier is null) and the
// two ascending lists to list[] as 16-bit column indices: full at [0, n_full), approximate at
// [a0, a0 + n_approx) with a0 = n_full rounded up to 4. Thread i owns the contiguous quads
// [i c, (i + 1) c): one block scan orders everything. Returns n_full, n_approx and a0 (identical
// in every thread); ends with a barrier, so list[] can be read at once.
__device__ __forceinline__ void select_compact(const uint32_t* __restrict__ keys, int d,
                                               const Boundary* B, SelectSmem& S,
                                               uint8_t* __restrict__ tier,
                                               uint16_t* __restrict__ list, uint32_t* n_full,
                                               uint32_t* n_approx, uint32_t* a0_out) {
  const int tid = threadIdx.x;
  const int nq = (d + 3) >> 2, nfull = d >> 2;
  const int cq = (nq + kSelThreads - 1) / kSelThreads;
  const int qa = min(nq, tid * cq), qb = min(nq, qa + cq);
  const int qm = max(qa, min(qb, nfull));  // quads [qa, qm) lie wholly inside d
  const uint4* kq = reinterpret_cast<const uint4*>(keys);
  const uint32_t lo0 = B[0].lo, lo1 = B[1].lo, ev0 = B[0].eqv, ev1 = B[1].eqv;
  const uint32_t rem0 = B[0].rem, rem1 = B[1].rem;
  const bool ties = ev0 != kNoKey || ev1 != kNoKey;
  const bool ragged = qm < qb;  // this thread owns the quad that d cuts
  const int lim = d - 4 * nfull;
  // ---- pass 3: counts over the run ----
  uint32_t g0 = 0, g1 = 0, e0 = 0, e1 = 0;
  for (int q = qa; q < qm; ++q) {
    const uint4 v = ld_key4(kq, q);
    g0 += (v.x >= lo0) + (v.y >= lo0) + (v.z >= lo0) + (v.w >= lo0);
    g1 += (v.x >= lo1) + (v.y >= lo1) + (v.z >= lo1) + (v.w >= lo1);
  }
  if (ragged) {
    const uint4 v = ld_key4(kq, nfull);
    const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (e < lim) g0 += kk[e] >= lo0, g1 += kk[e] >= lo1;
    }
  }
  uint32_t eb0 = 0, eb1 = 0, tot;
  if (ties) {  // keys equal to a boundary key before this run, in column order
    for (int q = qa; q < qb; ++q) {
      const uint4 v = ld_key4(kq, q);
      const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool ok = 4 * q + e < d;
        e0 += ok && kk[e] == ev0;
        e1 += ok && kk[e] == ev1;
      }
    }
    const uint32_t ex = block_excl_scan(e0 | (e1 << 16), S, &tot);
    eb0 = ex & 0xFFFFu;
    eb1 = ex >> 16;
    g0 += min(e0, rem0 > eb0 ? rem0 - eb0 : 0u);
    g1 += min(e1, rem1 > eb1 ? rem1 - eb1 : 0u);
  }
  // the last scan of the selection: nothing writes S.wscan before the closing barrier below
  const uint32_t ex = block_excl_scan<false>(g0 | ((g1 - g0) << 16), S, &tot);
  const uint32_t nf = tot & 0xFFFFu, na = tot >> 16, a0 = (nf + 3u) & ~3u;
  *n_full = nf;
  *n_approx = na;
  *a0_out = a0;
  // ---- pass 4: tier codes; list entries staged in shared memory ----
  uint32_t pf = ex & 0xFFFFu, pa = a0 + (ex >> 16);
  const uint32_t cap = (uint32_t)(select_list_bytes(d) / 2);  // entries; a guard, never reached
  const bool tier_vec = (reinterpret_cast<uintptr_t>(tier) & 3u) == 0;
  if (!ties) {
    for (int q = qa; q < qm; ++q) {
      const uint4 v = ld_key4(kq, q);
      const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
      uint32_t packed = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t f = kk[e] >= lo0, a = kk[e] >= lo1;  // f implies a
        const uint32_t at = f ? pf : pa;
        if (a && at < cap) list[at] = (uint16_t)(4 * q + e);
        pf += f;
        pa += a - f;
        packed |= (f + a) << (8 * e);
      }
      if (tier) {
        if (tier_vec) {
          reinterpret_cast<uint32_t*>(tier)[q] = packed;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) tier[4 * q + e] = (uint8_t)(packed >> (8 * e));
        }
      }
    }
  }
  if (__builtin_expect(ties || ragged, 0)) {  // the general form: bounds checks and ordered equal keys
    for (int q = ties ? qa : qm; q < qb; ++q) {
      const uint4 v = ld_key4(kq, q);
      const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (4 * q + e < d) {
          bool in0 = kk[e] >= lo0, in1 = kk[e] >= lo1;
          if (kk[e] == ev0) in0 = eb0++ < rem0;
          if (kk[e] == ev1) in1 = eb1++ < rem1;
          in1 = in1 || in0;
          const uint32_t at = in0 ? pf : pa;
          if (in1 && at < cap) list[at] = (uint16_t)(4 * q + e);
          pf += in0;
          pa += in1 && !in0;
          if (tier) tier[4 * q + e] = (uint8_t)((uint32_t)in0 + (uint32_t)in1);
        }
      }
    }
  }
  __syncthreads();
}

// Copy the staged lists to global memory as int32 (coalesced; 16-byte stores when the
// destinations allow). All threads.
__device__ __forceinline__ void select_write_lists(const uint16_t* __restrict__ list, int d,
                                                   uint32_t nf, uint32_t na, uint32_t a0,
                                                   int32_t* __restrict__ full_idx,
                                                   int32_t* __restrict__ approx_idx) {
  const int tid = threadIdx.x;
  if (nf + na > (uint32_t)d) return;  // a guard: the counts never exceed d
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const uint16_t* src = list + (t ? a0 : 0u);
    int32_t* dst = t ? approx_idx : full_idx;
    const uint32_t n = t ? na : nf;
    if ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
      for (uint32_t i = 4u * tid; i < n; i += 4u * kSelThreads) {
        const uint2 p = *reinterpret_cast<const uint2*>(src + i);
        if (i + 4u <= n) {
          *reinterpret_cast<int4*>(dst + i) =
              make_int4((int)(p.x & 0xFFFFu), (int)(p.x >> 16), (int)(p.y & 0xFFFFu), (int)(p.y >> 16));
        } else {
          const uint32_t w[4] = {p.x & 0xFFFFu, p.x >> 16, p.y & 0xFFFFu, p.y >> 16};
#pragma unroll
          for (uint32_t e = 0; e < 4; ++e)
            if (i + e < n) dst[i + e] = (int32_t)w[e];
        }
      }
    } else {
      for (uint32_t i = tid; i < n; i += kSelThreads) dst[i] = (int32_t)src[i];
    }
  }
}

}  // namespace spax
