// select_fused.cuh — the tier rule as the masked GEMV runs it in every CTA: the columns whose
// tier is certain after one histogram pass are sorted into this CTA's share at once, and only
// the columns of the two boundary bins are ranked further.
//
// Sources: SpAx (arXiv 2610.02598), Abstract — skip the columns whose activations are closest to
// zero, approximate the smaller ones, read the largest in full. TopK-Guided (arXiv 2610.01763),
// Abstract and §1 — the threshold rule (TEAL) and the fixed-count TopK rule (WINA); §2.1 — the
// natural sparsity from the calibrated threshold, clipped to a ±δ band around the target, then
// TopK. The rule, the rank order and the tie order are the ones select.cuh implements (larger |x|
// first, equal |x| by lower column first); only the order of the work differs.
//
// Steps (all threads of a 512-thread CTA; keys = x as fp32 bits in shared memory):
//   coarse   pass 1 of select.cuh (a 4096-bin histogram of key bits 30..19, the threshold counts,
//            the non-finite check) and the block-wide find: a TopK-type boundary t whose rank K_t
//            falls in bin p_t has the window [p_t << 19, (p_t + 1) << 19). Every key above a
//            window is certainly in, every key below it certainly out. A threshold-type boundary
//            is exact at once (an empty window at its threshold).
//   certain  one counting pass over contiguous per-thread runs of columns and one block scan:
//            the certain-full and certain-approximate columns in ascending order, of which this
//            CTA keeps the positions p with p mod S == split (at local index p / S), and the
//            candidates (keys inside a window) in ascending column order, which every CTA keeps.
//   resolve  select.cuh's passes 2 / 2b, over the candidates only: the boundary key V_t, the
//            number of keys above it and how many copies of V_t are in.
//   boundary the exact tiers of the candidates (equal keys at a boundary ranked by column), and
//            this CTA's share of the candidates that are in: the full list of the split is the
//            concatenation certain ++ boundary, position P of it at local index P / S.
//   outputs  the tier codes and the ascending lists, when asked for, by one CTA: an exact
//            compaction over all columns writing global memory.
#pragma once

#include "select.cuh"

namespace spax {

// p / S and p mod S for p < 2^16 and S <= 256 by one multiply: m = ceil(2^32 / S) (S == 1: m = 0,
// quotient p). floor(p m / 2^32) = floor(p / S) because p (m - 2^32 / S) / 2^32 < 2^-16 < 1 / S.
__host__ __device__ inline uint32_t split_magic(uint32_t S) {
  return S <= 1u ? 0u : (uint32_t)((0xFFFFFFFFull / S) + 1ull);
}
__device__ __forceinline__ uint32_t div_split(uint32_t p, uint32_t S, uint32_t m) {
  return m ? __umulhi(p, m) : p;
}

// The coarse stage: pass 1 and, for TopK-type boundaries, the bin of each rank K. Fills the two
// windows (clo, chi), the rank data of each TopK-type boundary (kind 2: K_t, the count above its
// bin, the bin), and the threshold counts n1, n2 (guided mode; 0 otherwise). Threshold mode runs
// no pass here (its non-finite check is made by the certain pass). Returns true on a non-finite
// key (TopK and guided modes). All threads; barriers inside; results identical in every thread.
struct Coarse {
  uint32_t clo[2], chi[2];  // candidates of boundary t: keys in [clo_t, chi_t)
  uint32_t K[2], above[2], bin[2];
  int kind[2];              // 0 empty, 1 exact (threshold or every column), 2 TopK rank in a bin
};

__device__ __forceinline__ bool fsel_coarse(const spax_mask_params& prm, int d,
                                            const uint32_t* __restrict__ keys, SelectSmem& S,
                                            uint32_t* n1, uint32_t* n2, Coarse& C) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const uint32_t ts = __float_as_uint(prm.t_skip) & 0x7FFFFFFFu;
  const uint32_t tf = __float_as_uint(prm.t_full) & 0x7FFFFFFFu;
  *n1 = *n2 = 0u;
  uint32_t lo[2] = {tf, ts};
  if (prm.mode == SPAX_MASK_THRESHOLD) {
    C.kind[0] = C.kind[1] = 1;
  } else {
    bool bad;
    select_pass1(prm.mode, d, ts, tf, keys, S, n1, n2, &bad);
    if (bad) return true;
    if (prm.mode == SPAX_MASK_TOPK) {
      C.K[0] = (uint32_t)prm.k_full;
      C.K[1] = (uint32_t)prm.k_full + (uint32_t)prm.k_approx;
      for (int t = 0; t < 2; ++t) {
        C.kind[t] = C.K[t] == 0u ? 0 : (C.K[t] >= (uint32_t)d ? 1 : 2);
        if (C.kind[t] == 1) lo[t] = 0u;  // every column
      }
    } else {  // guided: the band-clipped counts, exact when equal to the natural count
      const long long m1 = guided_clip(*n1, d, prm.s_skip_bp, prm.delta_bp);
      long long m2 = guided_clip(*n2, d, prm.s_below_full_bp, prm.delta_bp);
      if (m2 < m1) m2 = m1;
      C.K[0] = (uint32_t)(d - m2);
      C.K[1] = (uint32_t)(d - m1);
      const uint32_t nat[2] = {(uint32_t)d - *n2, (uint32_t)d - *n1};
      for (int t = 0; t < 2; ++t) {
        if (C.K[t] == nat[t]) C.kind[t] = 1;  // the threshold set itself
        else if (C.K[t] == 0u) C.kind[t] = 0;
        else if (C.K[t] >= (uint32_t)d) C.kind[t] = 1, lo[t] = 0u;
        else C.kind[t] = 2;
      }
    }
    if (C.kind[0] == 2 || C.kind[1] == 2) {
      // the 12-bit bins of ranks K0, K1: thread t owns bins 4095-8t .. 4088-8t (high to low)
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
      for (int g = 0; g < kSelWarps / 4; ++g) {
        const uint4 q = *reinterpret_cast<const uint4*>(&S.wsum[4 * g]);
        cum += (4 * g + 0 < wid ? q.x : 0u) + (4 * g + 1 < wid ? q.y : 0u) +
               (4 * g + 2 < wid ? q.z : 0u) + (4 * g + 3 < wid ? q.w : 0u);
      }
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const uint32_t K = C.K[t];
        if (C.kind[t] == 2 && cum < K && K <= cum + s) {
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
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (C.kind[t] == 2) {
          C.bin[t] = S.sel[t][0];
          C.above[t] = S.sel[t][1];
        }
      }
      __syncthreads();  // S.sel is rewritten by the resolve step
    }
  }
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (C.kind[t] == 2) {
      C.clo[t] = C.bin[t] << 19;
      C.chi[t] = (C.bin[t] + 1u) << 19;
    } else {
      const uint32_t l = C.kind[t] == 0 ? kNoLo : lo[t];
      C.clo[t] = C.chi[t] = l;
    }
  }
  return false;
}

// Class of one key after the coarse stage: a candidate (inside either window: every key of a
// window counts towards that boundary's rank, whatever the other boundary makes of it), else
// certainly full (above window 0), certainly approximate (above window 1 only) or skipped.
struct KeyClass {
  bool f, a, c;
};
__device__ __forceinline__ KeyClass classify(uint32_t k, const Coarse& C) {
  KeyClass r;
  r.c = (k - C.clo[0] < C.chi[0] - C.clo[0]) || (k - C.clo[1] < C.chi[1] - C.clo[1]);
  r.f = !r.c && k >= C.chi[0];
  r.a = !r.c && !r.f && k >= C.chi[1];
  return r;
}

// Exclusive block-wide prefix of two packed words per thread (16-bit fields), in thread order;
// scratch holds 2 x kSelWarps words. Totals in *t0, *t1. Two barriers; scratch reusable after.
__device__ __forceinline__ uint2 block_excl_scan2(uint32_t v0, uint32_t v1, uint32_t* scratch,
                                                  uint32_t* t0, uint32_t* t1) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t i0 = v0, i1 = v1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n0 = __shfl_up_sync(0xffffffffu, i0, o);
    const uint32_t n1 = __shfl_up_sync(0xffffffffu, i1, o);
    if (lane >= o) i0 += n0, i1 += n1;
  }
  if (lane == 31) scratch[wid] = i0, scratch[kSelWarps + wid] = i1;
  __syncthreads();
  uint32_t b0 = 0, b1 = 0, a0 = 0, a1 = 0;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) {
    const uint32_t s0 = scratch[w], s1 = scratch[kSelWarps + w];
    b0 += w < wid ? s0 : 0u;
    b1 += w < wid ? s1 : 0u;
    a0 += s0;
    a1 += s1;
  }
  __syncthreads();
  *t0 = a0;
  *t1 = a1;
  return make_uint2(b0 + i0 - v0, b1 + i1 - v1);
}

// The certain step. Thread i owns the contiguous quads [i cq, (i + 1) cq). Writes this CTA's
// share of the certain-full / certain-approximate columns (ascending position p, kept when
// p mod S == split, at index p / S of lf / la; at most cap entries each) and every candidate in
// ascending column order to cand[] (at most d entries). Returns the totals (block-uniform) and
// whether a key was non-finite. All threads; barriers inside; ends with a barrier.
__device__ __forceinline__ void fsel_certain(const uint32_t* __restrict__ keys, int d,
                                             const Coarse& C, uint32_t S, uint32_t split,
                                             uint32_t smagic, uint16_t* __restrict__ lf,
                                             uint16_t* __restrict__ la, uint32_t cap,
                                             uint16_t* __restrict__ cand, SelectSmem& sm,
                                             uint32_t* nCF, uint32_t* nCA, uint32_t* nC,
                                             bool* bad) {
  const int tid = threadIdx.x;
  const int nq = (d + 3) >> 2;
  const int cq = (nq + kSelThreads - 1) / kSelThreads;
  const int qa = min(nq, tid * cq), qb = min(nq, qa + cq);
  const uint4* kq = reinterpret_cast<const uint4*>(keys);
  uint32_t cf = 0, ca = 0, cc = 0, nb = 0;
  for (int q = qa; q < qb; ++q) {
    const uint4 v = ld_key4(kq, q);
    const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (4 * q + e < d) {
        const KeyClass r = classify(kk[e], C);
        cf += r.f;
        ca += r.a;
        cc += r.c;
        nb |= kk[e] >= 0x7F800000u;
      }
    }
  }
  uint32_t tot0, tot1;
  const uint2 ex = block_excl_scan2(cf | (ca << 16), cc | (nb << 16), sm.wscan2, &tot0, &tot1);
  *nCF = tot0 & 0xFFFFu;
  *nCA = tot0 >> 16;
  *nC = tot1 & 0xFFFFu;
  *bad = (tot1 >> 16) != 0u;
  if (*bad) return;  // block-uniform
  uint32_t pf = ex.x & 0xFFFFu, pa = ex.x >> 16, pc = ex.y & 0xFFFFu;
  for (int q = qa; q < qb; ++q) {
    const uint4 v = ld_key4(kq, q);
    const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t j = 4u * q + e;
      if (j < (uint32_t)d) {
        const KeyClass r = classify(kk[e], C);
        if (r.f) {
          const uint32_t i = div_split(pf, S, smagic);
          if (pf - i * S == split && i < cap) lf[i] = (uint16_t)j;
          ++pf;
        } else if (r.a) {
          const uint32_t i = div_split(pa, S, smagic);
          if (pa - i * S == split && i < cap) la[i] = (uint16_t)j;
          ++pa;
        } else if (r.c) {
          cand[pc++] = (uint16_t)j;
        }
      }
    }
  }
  __syncthreads();
}

// The resolve step: for each TopK-type boundary t, the key V_t of rank K_t, found among the
// candidates inside its window (select.cuh's pass 2 over key bits 18..9 and, when rank K_t is
// not the last key of its sub-bin, pass 2b over bits 8..0). Sets B[t] for every boundary. All
// threads; barriers inside; B identical in every thread.
__device__ __forceinline__ void fsel_resolve(const uint32_t* __restrict__ keys,
                                             const uint16_t* __restrict__ cand, uint32_t ncand,
                                             const Coarse& C, SelectSmem& S, Boundary* B) {
  const int tid = threadIdx.x;
  const bool sel0 = C.kind[0] == 2, sel1 = C.kind[1] == 2;
  uint32_t V[2] = {0u, 0u}, ab[2] = {0u, 0u}, cnt[2] = {0u, 0u};
  if (sel0 || sel1) {
    const uint32_t p0 = sel0 ? C.bin[0] : kNoKey, p1 = sel1 ? C.bin[1] : kNoKey;
    const bool same = p0 == p1;
    for (uint32_t i = tid; i < ncand; i += kSelThreads) {
      const uint32_t k = keys[cand[i]] & 0x7FFFFFFFu, b = k >> 19;
      if (b == p0 || b == p1) atomicAdd(&S.ha[b == p0 ? 0 : 1][(k >> 9) & 1023u], 1u);
    }
    __syncthreads();
    block_find_pair<1024>(S.ha[0], same ? S.ha[0] : S.ha[1], sel0, sel1, C.K[0], C.K[1],
                          C.above[0], C.above[1], p0, p1, 10, S);
    bool need[2] = {false, false};
    uint32_t q[2] = {kNoKey, kNoKey};
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (C.kind[t] != 2) continue;
      const uint32_t pre = S.sel[t][0], above = S.sel[t][1], c = S.sel[t][2];
      if (C.K[t] - above == c) {  // all of the sub-bin: its smallest key bounds the set
        V[t] = pre << 9;
        ab[t] = above;
        cnt[t] = kNoKey;
      } else {
        need[t] = true;
        q[t] = pre;
      }
    }
    if (need[0] || need[1]) {
      const uint32_t abA0 = S.sel[0][1], abA1 = S.sel[1][1];
      __syncthreads();  // S.sel is rewritten below
      const bool same2 = q[0] == q[1];
      for (uint32_t i = tid; i < ncand; i += kSelThreads) {
        const uint32_t k = keys[cand[i]] & 0x7FFFFFFFu, b = k >> 9;
        if (b == q[0] || b == q[1]) atomicAdd(&S.hb[b == q[0] ? 0 : 1][k & 511u], 1u);
      }
      __syncthreads();
      block_find_pair<512>(S.hb[0], same2 ? S.hb[0] : S.hb[1], need[0], need[1], C.K[0], C.K[1],
                           abA0, abA1, q[0], q[1], 9, S);
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (need[t]) V[t] = S.sel[t][0], ab[t] = S.sel[t][1], cnt[t] = S.sel[t][2];
    }
  }
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (C.kind[t] == 2) {
      const uint32_t rem = C.K[t] - ab[t];
      if (cnt[t] == kNoKey || rem == cnt[t]) {
        B[t].lo = V[t];
        B[t].eqv = kNoKey;
        B[t].rem = 0u;
      } else {
        B[t].lo = V[t] + 1u;
        B[t].eqv = V[t];
        B[t].rem = rem;
      }
    } else {
      B[t].lo = C.clo[t];  // exact: threshold, every column (0) or none (kNoLo)
      B[t].eqv = kNoKey;
      B[t].rem = 0u;
    }
  }
}

// The boundary step: the exact tiers of the candidates (ascending columns; keys equal to a
// boundary key ranked by column) and this CTA's share of those that are in, appended to lf / la
// at global positions nCF + i / nCA + i of the concatenated lists. Returns the boundary counts
// (block-uniform). All threads; barriers inside; ends with a barrier.
__device__ __forceinline__ void fsel_boundary(const uint32_t* __restrict__ keys,
                                              const uint16_t* __restrict__ cand, uint32_t ncand,
                                              const Boundary* B, uint32_t nCF, uint32_t nCA,
                                              uint32_t S, uint32_t split, uint32_t smagic,
                                              uint16_t* __restrict__ lf, uint16_t* __restrict__ la,
                                              uint32_t cap, SelectSmem& sm, uint32_t* nBF,
                                              uint32_t* nBA) {
  const int tid = threadIdx.x;
  const uint32_t cc = (ncand + kSelThreads - 1) / kSelThreads;
  const uint32_t ia = min(ncand, tid * cc), ib = min(ncand, ia + cc);
  const uint32_t lo0 = B[0].lo, lo1 = B[1].lo, ev0 = B[0].eqv, ev1 = B[1].eqv;
  const uint32_t rem0 = B[0].rem, rem1 = B[1].rem;
  const bool ties = ev0 != kNoKey || ev1 != kNoKey;
  uint32_t eb0 = 0, eb1 = 0, tot0, tot1;
  if (ties) {  // keys equal to a boundary key before this run (every such key is a candidate)
    uint32_t e0 = 0, e1 = 0;
    for (uint32_t i = ia; i < ib; ++i) {
      const uint32_t k = keys[cand[i]] & 0x7FFFFFFFu;
      e0 += k == ev0;
      e1 += k == ev1;
    }
    const uint2 ex = block_excl_scan2(e0, e1, sm.wscan2, &tot0, &tot1);
    eb0 = ex.x;
    eb1 = ex.y;
  }
  uint32_t bf = 0, ba = 0;
  {
    uint32_t f0 = eb0, f1 = eb1;
    for (uint32_t i = ia; i < ib; ++i) {
      const uint32_t k = keys[cand[i]] & 0x7FFFFFFFu;
      bool in0 = k >= lo0, in1 = k >= lo1;
      if (k == ev0) in0 = f0++ < rem0;
      if (k == ev1) in1 = f1++ < rem1;
      in1 = in1 || in0;
      bf += in0;
      ba += in1 && !in0;
    }
  }
  const uint2 ex = block_excl_scan2(bf, ba, sm.wscan2, &tot0, &tot1);
  *nBF = tot0;
  *nBA = tot1;
  uint32_t pf = nCF + ex.x, pa = nCA + ex.y;
  for (uint32_t i = ia; i < ib; ++i) {
    const uint32_t j = cand[i], k = keys[j] & 0x7FFFFFFFu;
    bool in0 = k >= lo0, in1 = k >= lo1;
    if (k == ev0) in0 = eb0++ < rem0;
    if (k == ev1) in1 = eb1++ < rem1;
    in1 = in1 || in0;
    if (in0) {
      const uint32_t q = div_split(pf, S, smagic);
      if (pf - q * S == split && q < cap) lf[q] = (uint16_t)j;
      ++pf;
    } else if (in1) {
      const uint32_t q = div_split(pa, S, smagic);
      if (pa - q * S == split && q < cap) la[q] = (uint16_t)j;
      ++pa;
    }
  }
  __syncthreads();
}

// The optional outputs in ascending order, by one CTA: tier codes (may be null) and both lists
// (either may be null) as spax_build_mask writes them, from the exact boundaries B. Thread i owns
// the contiguous quads [i cq, (i + 1) cq); a tie scan first when a boundary key is cut. scratch:
// 2 x kSelWarps words of its own. All threads; barriers inside.
__device__ __forceinline__ void fsel_write_outputs(const uint32_t* __restrict__ keys, int d,
                                                   const Boundary* B, uint32_t* scratch,
                                                   uint8_t* __restrict__ tier,
                                                   int32_t* __restrict__ fidx,
                                                   int32_t* __restrict__ aidx) {
  const int tid = threadIdx.x;
  const int nq = (d + 3) >> 2;
  const int cq = (nq + kSelThreads - 1) / kSelThreads;
  const int qa = min(nq, tid * cq), qb = min(nq, qa + cq);
  const uint4* kq = reinterpret_cast<const uint4*>(keys);
  const uint32_t lo0 = B[0].lo, lo1 = B[1].lo, ev0 = B[0].eqv, ev1 = B[1].eqv;
  const uint32_t rem0 = B[0].rem, rem1 = B[1].rem;
  const bool ties = ev0 != kNoKey || ev1 != kNoKey;
  uint32_t eb0 = 0, eb1 = 0, tot0, tot1;
  if (ties) {
    uint32_t e0 = 0, e1 = 0;
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
    const uint2 ex = block_excl_scan2(e0, e1, scratch, &tot0, &tot1);
    eb0 = ex.x;
    eb1 = ex.y;
  }
  uint32_t nf = 0, na = 0;
  {
    uint32_t f0 = eb0, f1 = eb1;
    for (int q = qa; q < qb; ++q) {
      const uint4 v = ld_key4(kq, q);
      const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (4 * q + e < d) {
          bool in0 = kk[e] >= lo0, in1 = kk[e] >= lo1;
          if (kk[e] == ev0) in0 = f0++ < rem0;
          if (kk[e] == ev1) in1 = f1++ < rem1;
          in1 = in1 || in0;
          nf += in0;
          na += in1 && !in0;
        }
      }
    }
  }
  const uint2 ex = block_excl_scan2(nf, na, scratch, &tot0, &tot1);
  uint32_t pf = ex.x, pa = ex.y;
  for (int q = qa; q < qb; ++q) {
    const uint4 v = ld_key4(kq, q);
    const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * q + e;
      if (j < d) {
        bool in0 = kk[e] >= lo0, in1 = kk[e] >= lo1;
        if (kk[e] == ev0) in0 = eb0++ < rem0;
        if (kk[e] == ev1) in1 = eb1++ < rem1;
        in1 = in1 || in0;
        if (in0 && fidx) fidx[pf] = j;
        if (in1 && !in0 && aidx) aidx[pa] = j;
        pf += in0;
        pa += in1 && !in0;
        if (tier) tier[j] = (uint8_t)((uint32_t)in0 + (uint32_t)in1);
      }
    }
  }
}

}  // namespace spax
