// gemv.cu — the fused tiered gather-GEMV (and the dense bf16 GEMV built from the same kernel).
//
// y = Σ_{j in full} x_j W[:,j] + Σ_{j in approx} x_j (min_g + q·scale_g)[:,j]   (fp32 accumulate)
//
// Sources: SpAx (arXiv 2610.02598), Abstract — original weights for the largest |x|,
// approximate weights for smaller |x|, nothing for the rest; eigenradar commentary on SpAx,
// "The route outside GPU memory" — cost is bytes moved per token plus the time to reconstruct
// the two-bit approximations on the GPU.
//
// Design (B200, HBM-bound; no tensor cores — a batch-one GEMV has no reuse):
//   * Grid = T row tiles (R = 512*RG rows) x S column splits, one CTA of 16 warps per SM (single
//     wave). Split s takes positions s, s+S, s+2S, ... of the compacted approx list and of the
//     full list, so every CTA gets the same mix of byte-heavy (bf16/int4) and ALU-heavy (2-bit)
//     columns and the S CTAs of a tile sweep neighbouring columns together. The positions do not
//     depend on the counts, so the index loads are issued together with the device-side counts
//     load (one memory round trip, no host sync).
//   * Warp (rg, cg) owns rows [512 rg, 512 rg + 512) of the tile and every CG-th column of the
//     CTA's share. Lane l owns rows 8l..8l+7 and 256+8l..256+8l+7 in all three formats, so bf16,
//     int4 and 2-bit contributions land in the same 16 fp32 accumulators. Weights stream straight
//     into registers with 16-byte loads marked evict-first, U bf16 columns in flight per warp;
//     the small 2-bit and int4 records come by cp.async into a per-warp double buffer in shared
//     memory, each batch sent one batch ahead. A warp's short last bf16 round is fetched into
//     the idle second buffer with the first loads.
//     (Measured on B200: one-warp-issued 1-D bulk copies of 0.1-4 KB column segments are
//     issue-bound at 0.5-3 TB/s; plain 16-byte loads from many warps reach 6.4-6.9 TB/s.)
//   * 2-bit and int4 codes become floats with one LOP3 each: the code is masked into the
//     mantissa of a power-of-two constant C (value C + q exactly), multiplied by x_j*scale and
//     the constant's contribution C*Σ x_j*scale is removed once per row at the end.
//   * Warps' partial rows are combined in shared memory in a fixed order. Split-K partials go to
//     the workspace as 64-bit words that carry the value and a ready flag together (one
//     single-copy-atomic store: no fence and no arrival counter on the critical path); each of
//     the S CTAs of a tile then sums one slice of the tile's rows over the S splits in split
//     order (bit-reproducible) and clears the words it read. The grid is one wave, so the CTAs
//     that wait for one another are all resident; the wait is bounded (SPAX_ERR_TIMEOUT).
#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace spax {

constexpr int kGemvWarps = 16;
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kGemvMeta = 1024;  // metadata slots per list per chunk
constexpr int kGemvU = 4;        // columns in flight per warp

// Small records (2-bit: 144 B per column and 512 rows; int4: 272 B per column and 512 rows) are
// fetched a batch at a time by cp.async into a per-warp double buffer (16-byte pieces), the next
// batch in flight while the current one is decoded, so a warp keeps 2-4 KB in flight instead of a
// few bytes per lane.
constexpr int kBatch2 = 16;                // 2-bit columns per staged batch
constexpr int kBatch4 = 8;                 // int4 columns per staged batch (two in flight)
constexpr int kStage2Bytes = 16 * 144;      // one batch of 2-bit records
constexpr int kStageRecBytes = 2 * kStage2Bytes;  // two 2-bit batches (>= one int4 batch, 16 * 272)
constexpr int kStageWarpBytes = kStageRecBytes + 16 * 32;  // + 4 coefficient pairs per column

// Row tile of R = 512 RG rows (RG = 1, 2 or 4, a launch parameter): warp (rg, cg) takes rows
// [512 rg, 512 rg + 512) of the tile and every CG-th column of the CTA's share, CG = 16 / RG.
// One kernel image serves every tile height, so the launches of a decoder layer (whose shapes
// want different tiles) all run the same code and keep it warm in the instruction caches.
constexpr int kCombineFloats = kGemvWarps * 576;  // CG slots of (R / 32) * 36 floats, any RG
constexpr size_t kGemvSmemBytes = size_t(2) * kGemvMeta * 4 + size_t(kCombineFloats) * 4 +
                                  size_t(kGemvWarps) * kStageWarpBytes;
constexpr int kStage4Bytes = kBatch4 * 272;  // one batch of int4 half-records
static_assert(2 * kStage4Bytes <= kStageRecBytes && 2 * kBatch2 * 144 <= kStageRecBytes, "staging");

struct GemvParams {
  const uint8_t* full;
  const uint8_t* approx;
  const float* x;
  const int32_t* fidx;
  const int32_t* aidx;
  const int32_t* counts;
  float* y;
  unsigned long long* part;  // [S][d_out] flagged partial sums, zero at rest
  int32_t* status;
  long long full_col_stride;    // bytes between full-pool columns
  long long approx_col_stride;  // bytes between approx-pool columns
  int d_out, d_in, S;
  // fused mask (masked GEMV only): the rule, the optional outputs, the staged-list bytes
  spax_mask_params prm;
  uint8_t* tier_out;
  int32_t* fidx_out;
  int32_t* aidx_out;
  int32_t* counts_out;
  int list_bytes;  // 0 for the list-driven kernels
  int keys_bytes;  // fused: x kept alive after the lists for the product (0: x shares the reused
                   // area with the GEMV's staging, and the kernel stashes its split's x values)
  int RG;          // row tile R = 512 * RG (1, 2 or 4)
  float* x_out;    // fused swiglu only: the token's x (lead CTA; may be null)
  const float* norms;  // fused only, may be null: rank by the WINA score |x_j| * norms[j]
  int fetch_swiglu;    // plain instance only: x is formed from [g; u] (every x the product needs
                       // is then in shared memory: the host checks)
  unsigned long long wait_ns;  // bound of the split-K wait
};

// Code -> float: (word & (mask << p)) | bits(C) is the float C + code, exactly, when C = 2^(23-p)
// (the code lands in the mantissa bits whose weight is 1). Written as one LOP3 with the mask
// immediate and bits(C) in a register: with both operands immediate the compiler splits it into
// two integer-pipe instructions (measured: 32 instead of 16 per 512-row 2-bit column segment).
template <uint32_t MASK>
__device__ __forceinline__ float code_f(uint32_t rot, uint32_t c_bits) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(rot), "n"(MASK), "r"(c_bits));  // (a&b)|c
  return __uint_as_float(d);
}
// bits(C) for C = 256, 64, 16, 4, held in registers (an opaque move keeps the compiler from
// folding them back into immediates)
__device__ __forceinline__ uint32_t reg_const(uint32_t v) {
  uint32_t r;
  asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v));
  return r;
}

// Index of row r inside a combine slot (36 floats per 32 rows: padding spreads the banks).
__device__ __forceinline__ int red_row(int r) { return (r >> 5) * 36 + (r & 31); }

__device__ __forceinline__ uint4 ld_stream128(const uint8_t* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ uint32_t ld_stream32(const uint8_t* p) {
  return __ldcs(reinterpret_cast<const unsigned int*>(p));
}
__device__ __forceinline__ uint32_t ld_stream16(const uint8_t* p) {
  return __ldcs(reinterpret_cast<const unsigned short*>(p));
}

// ---- flagged partial sums: (value bits | 1 << 32) per 64-bit word; 0 means "not written" ----
__device__ __forceinline__ void st_ll4(unsigned long long* p, float4 v) {
  const unsigned long long f = 1ull << 32;
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(p),
               "l"(f | __float_as_uint(v.x)), "l"(f | __float_as_uint(v.y))
               : "memory");
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(p + 2),
               "l"(f | __float_as_uint(v.z)), "l"(f | __float_as_uint(v.w))
               : "memory");
}
// The four words at p, when all four carry their flag.
__device__ __forceinline__ bool ld_ll4(const unsigned long long* p, float4* v) {
  unsigned long long a, b, c, d;
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(c), "=l"(d) : "l"(p + 2) : "memory");
  if (((a & b & c & d) >> 32) == 0) return false;  // a flag is the word's only high bit
  *v = make_float4(__uint_as_float((uint32_t)a), __uint_as_float((uint32_t)b),
                   __uint_as_float((uint32_t)c), __uint_as_float((uint32_t)d));
  return true;
}
__device__ __forceinline__ void clear_ll4(unsigned long long* p) {
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %1};" ::"l"(p), "l"(0ull) : "memory");
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %1};" ::"l"(p + 2), "l"(0ull) : "memory");
}

// Shared memory of the fused kernel ahead of the GEMV's own areas: the selection's scratch and
// keys share space with the combine and staging areas (they are dead before the GEMV starts).
__host__ __device__ inline size_t fused_select_bytes(int d) {
  return (sizeof(SelectSmem) + 15) / 16 * 16 + select_keys_bytes(d);
}

// FUSED, the mask of the launch: 0 for the list-driven and dense kernels, which take their lists
// from the caller. Otherwise the kernel first runs the tier rule itself (select.cuh: every CTA
// computes the same lists, staged in its shared memory), then reads its split's positions from
// there. The rule runs on x (kFusedX), on x = silu(g) * u formed from [g; u] (kFusedSwiglu), or on
// the WINA score |x| * norm (kFusedScored). Each source is its own instance: code in this kernel
// costs time even where it never runs (measured on the Llama-2-7B block: the plain instance 1.0 us
// per token-layer faster without the other two sources' code). The plain instance also serves the
// SwiGLU calls whose product finds every x in shared memory (it forms x in its fetch), so a decoder
// layer's launches share one image that stays warm in the instruction caches (measured: the layer
// with down fed from gate/up 68.8 -> 65.2 us); the SwiGLU instance serves the rest.
constexpr int kFusedX = 1, kFusedSwiglu = 2, kFusedScored = 3;
// Added to a source: the rule is TOPK_SCALED (the guesses of the boundary keys scale with the
// token's mean key), its own instances so that the others carry none of its code.
constexpr int kFusedScaled = 4;

// RGT: the row-tile factor fixed at compile time (1, 2, 4), or 0 for the launch's p.RG. The tiered
// kernels take 0 (one image for every shape of a layer); the dense baseline, a pure stream that
// gains from the constant, keeps one image per tile height.
template <int RGT, int FMT, bool DENSE, int FUSED>
__global__ void __launch_bounds__(kGemvThreads, 1) tiered_gemv_kernel(const GemvParams p) {
  constexpr int U = kGemvU;
  constexpr bool kSwiglu = (FUSED & 3) == kFusedSwiglu, kScored = (FUSED & 3) == kFusedScored;
  constexpr bool kScaled = (FUSED & kFusedScaled) != 0;
  const int RG = RGT > 0 ? RGT : p.RG, R = 512 * RG, CG = kGemvWarps / RG;
  const int kSlotFloats = RG * 576;  // combine slot of a column group: 36 floats per 32 rows
  static_assert(FMT == SPAX_FULL_BF16 || !DENSE, "the dense GEMV reads the bf16 pool");
  static_assert(!(DENSE && FUSED), "the dense GEMV has no mask");
  extern __shared__ __align__(128) uint8_t smem[];
  int32_t* meta_col_a = reinterpret_cast<int32_t*>(smem);
  int32_t* meta_col_f = meta_col_a + kGemvMeta;
  uint16_t* list = reinterpret_cast<uint16_t*>(meta_col_f + kGemvMeta);  // FUSED: staged lists
  float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(list) + p.list_bytes +
                                        p.keys_bytes);
  // fused, keys kept alive: x of every column for the product (null otherwise)
  const uint32_t* x_live = (FUSED && !kScored && p.keys_bytes)
                               ? reinterpret_cast<const uint32_t*>(reinterpret_cast<uint8_t*>(list) +
                                                                   p.list_bytes)
                               : nullptr;
  __shared__ int s_bad, s_last;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, split = blockIdx.y, S = p.S;
  // the decode constants (none in the dense GEMV)
  const uint32_t kC256 = DENSE ? 0u : reg_const(0x43800000u), kC64 = DENSE ? 0u : reg_const(0x42800000u);
  const uint32_t kC16 = DENSE ? 0u : reg_const(0x41800000u), kC4 = DENSE ? 0u : reg_const(0x40800000u);
  const int r0 = tile * R;
  const int rows_here = min(R, p.d_out - r0);
  const int rg = warp / CG, cg = warp % CG;
  const int rb = r0 + 512 * rg;              // first row of this warp
  const bool wrows = rb < p.d_out;           // the warp has rows (ragged last tile)
  const bool v0 = rb + 8 * lane < p.d_out;   // lane's first 8-row chunk is inside the matrix
  const bool v1 = rb + 256 + 8 * lane < p.d_out;
  // per-warp staging buffer: kBatch records, then their coefficients x*scale per 128-row group
  uint8_t* stage = reinterpret_cast<uint8_t*>(red + kCombineFloats) + warp * kStageWarpBytes;
  const uint32_t stage_s = smem_u32(stage);
  const uint32_t coef_s = stage_s + kStageRecBytes;

  if (tid == 0) {
    s_bad = 0;
    s_last = 0;
  }
  int Kf, Ka;
  uint32_t a0 = 0;  // FUSED: start of the approximate list in list[]
  if constexpr (FUSED) {
    // ---- the tier rule of this token, computed by every CTA (identical results) ----
    SelectSmem& sel = *reinterpret_cast<SelectSmem*>(red);
    uint32_t* keys = p.keys_bytes ? reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(list) +
                                                                 p.list_bytes)
                                  : reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(red) +
                                                 (sizeof(SelectSmem) + 15) / 16 * 16);
    select_zero(sel);
    pdl_wait();
    pdl_launch_dependents();
    float x_mean = -1.f;  // TOPK_SCALED on plain x: the mean |x| gathered by the fetch
    (void)x_mean;
    if constexpr (kSwiglu)
      select_fetch_swiglu(p.x, p.d_in, keys, tile == 0 && split == 0 ? p.x_out : nullptr);
    else if constexpr (kScored)
      select_fetch_scored(p.x, p.norms, p.d_in, keys);
    else if (p.fetch_swiglu)
      select_fetch_swiglu(p.x, p.d_in, keys, tile == 0 && split == 0 ? p.x_out : nullptr);
    else if constexpr (kScaled)
      x_mean = select_fetch_mean(p.x, p.d_in, keys, sel);  // the mean comes with the fetch
    else
      select_fetch(p.x, p.d_in, keys);
    uint32_t n1, n2;
    Boundary B[2];
    bool bad;
    if constexpr (kScaled)
      bad = select_rule(x_mean >= 0.f ? scaled_topk_params(p.prm, x_mean)
                                      : select_scaled_topk(p.prm, p.d_in, keys, sel),
                        p.d_in, keys, sel, &n1, &n2, B);
    else
      bad = select_rule(p.prm, p.d_in, keys, sel, &n1, &n2, B);
    const bool lead = tile == 0 && split == 0;
    if (__builtin_expect(bad, 0)) {  // non-finite x: every tier 0, empty lists, y = 0
      Kf = 0;
      Ka = 0;
      if (lead) {
        if (p.tier_out)
          for (int j = tid; j < p.d_in; j += kGemvThreads) p.tier_out[j] = 0;
        if (tid == 0) {
          if (p.counts_out) p.counts_out[0] = p.counts_out[1] = p.counts_out[2] = p.counts_out[3] = 0;
          record_status(p.status, SPAX_ERR_NONFINITE);
        }
      }
      __syncthreads();  // the selection's scratch is dead before the combine area reuses it
    } else {
      uint32_t nfu, nau;
      select_compact(keys, p.d_in, B, sel, lead ? p.tier_out : nullptr, list, &nfu, &nau, &a0);
      Kf = (int)nfu;
      Ka = (int)nau;
      if (tile == 0) {  // the tile-0 CTAs write the lists, each its own positions
        const int step = S * kGemvThreads;
        if (p.fidx_out)
          for (int q = split + S * tid; q < Kf; q += step) p.fidx_out[q] = list[q];
        if (p.aidx_out)
          for (int q = split + S * tid; q < Ka; q += step) p.aidx_out[q] = list[a0 + q];
        if (lead && tid == 0 && p.counts_out) {
          p.counts_out[0] = Kf;
          p.counts_out[1] = Ka;
          p.counts_out[2] = p.prm.mode == SPAX_MASK_TOPK ? 0 : (int32_t)n1;
          p.counts_out[3] = p.prm.mode == SPAX_MASK_TOPK ? 0 : (int32_t)n2;
        }
      }
      if (!p.keys_bytes) {
        // x shares the reused area: stash x of this split's first kGemvMeta positions of each
        // list in the metadata arrays (idle in this kernel) for the product (not with the WINA
        // score: its keys are scores, so the product reads x itself)
        const int nfl = kScored ? 0 : min(kGemvMeta, Kf > split ? (Kf - split + S - 1) / S : 0);
        const int nal = kScored ? 0 : min(kGemvMeta, Ka > split ? (Ka - split + S - 1) / S : 0);
        for (int i = tid; i < nfl; i += kGemvThreads)
          reinterpret_cast<float*>(meta_col_f)[i] = __uint_as_float(keys[list[split + S * i]]);
        for (int i = tid; i < nal; i += kGemvThreads)
          reinterpret_cast<float*>(meta_col_a)[i] = __uint_as_float(keys[list[a0 + split + S * i]]);
        __syncthreads();  // the keys are dead from here: the GEMV's staging areas reuse them
      }
    }
  } else {
    pdl_wait();
    pdl_launch_dependents();
  }

  // ---- counts and (speculatively) this split's first kGemvMeta positions of both lists ----
  if constexpr (FUSED) {
  } else if (DENSE) {
    Kf = p.d_in;
    Ka = 0;
  } else {
    Kf = __ldcg(p.counts);
    Ka = __ldcg(p.counts + 1);
    for (int i = tid; i < kGemvMeta; i += kGemvThreads) {
      const long long pos = split + (long long)S * i;
      if (pos < p.d_in) {
        meta_col_a[i] = __ldcg(p.aidx + pos);
        meta_col_f[i] = __ldcg(p.fidx + pos);
      }
    }
    if (Kf < 0 || Ka < 0 || Kf > p.d_in || Ka > p.d_in - Kf) {
      if (tid == 0) record_status(p.status, SPAX_ERR_INDEX);
      Kf = 0;
      Ka = 0;
    }
  }
  const int nf = Kf > split ? (Kf - split + S - 1) / S : 0;  // items of this split
  const int na = Ka > split ? (Ka - split + S - 1) / S : 0;
  const int nchunks = FUSED ? ((nf | na) ? 1 : 0) : (max(nf, na) + kGemvMeta - 1) / kGemvMeta;

  // this warp's slice of the packed pools
  const long long off_full = 2LL * (rb + 8 * lane);  // bf16 pool
  const long long off_approx = (long long)(rb / 512) * 144;
  const long long nib0 = (long long)(rb / 1024) * 528 + ((rb / 512) & 1) * 256;  // int4 pool
  const long long scl0 = (long long)(rb / 1024) * 528 + 512;
  const int half4 = (rb / 512) & 1;  // which half of its 1024-row int4 record the warp reads

  f2 acc[8];  // rows 8l..8l+7 (acc[0..3]) and 256+8l..256+8l+7 (acc[4..7]), as pairs
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = f2{0.f, 0.f};
  // per 128-row group g of the warp's 512 rows, summed over the columns this lane prepared:
  // 2-bit Σ x*scale and Σ x*min, int4 Σ x*scale (reduced over the warp at the end)
  float sA[4] = {0.f, 0.f, 0.f, 0.f}, bA[4] = {0.f, 0.f, 0.f, 0.f}, s4[4] = {0.f, 0.f, 0.f, 0.f};

  // x_j of a selected column (the fused swiglu kernel forms it from g_j and u_j again, with the
  // same function the selection used)
  auto xval = [&](int col) -> float {
    if constexpr (FUSED) {
      if constexpr (kSwiglu) return swiglu_x(__ldg(p.x + col), __ldg(p.x + p.d_in + col));
    }
    return __ldg(p.x + col);
  };

  // x of local position i of this split's approximate / full list: the fused kernel's stash
  // (first kGemvMeta positions), else x of the column
  const int xs_lim = (FUSED && !kScored && !p.keys_bytes) ? kGemvMeta : 0;  // stash positions
  auto xA = [&](int i, int col) -> float {
    if constexpr (FUSED) {
      if (x_live) return __uint_as_float(x_live[col]);
      if (i < xs_lim) return reinterpret_cast<const float*>(meta_col_a)[i];
    }
    return xval(col);
  };
  auto xF = [&](int i, int col) -> float {
    if constexpr (FUSED) {
      if (x_live) return __uint_as_float(x_live[col]);
      if (i < xs_lim) return reinterpret_cast<const float*>(meta_col_f)[i];
    }
    return xval(col);
  };

  // Column of local position i of this split's approximate / full list (in the current chunk):
  // the fused kernel reads its staged lists directly, the list-driven one its metadata arrays.
  auto colA = [&](int i) -> int {
    if constexpr (FUSED) return (int)list[a0 + split + S * i];
    else return meta_col_a[i];
  };
  auto colF = [&](int i) -> int {
    if constexpr (FUSED) return (int)list[split + S * i];
    else return meta_col_f[i];
  };

  // 2-bit column k of the staged batch: a lane's 8 rows in 16 bits, row i at bits 2i. Shifts left
  // by 15 and 7 (multiplies, which the FMA pipe can take) bring rows 0-3 and 4-7 to mantissa bits
  // 15, 17, 19, 21: values 256+q, 64+q, 16+q, 4+q. The coefficient comes as a ready pair.
  auto decode_approx = [&](int k, int buf = 0) {
    const uint32_t rec = stage_s + kStage2Bytes * buf + 144 * k;
    const uint32_t q01 = lds_u16(rec + 2 * lane);  // rows 8l .. 8l+7
    const uint32_t q11 = lds_u16(rec + 64 + 2 * lane);  // rows 256+8l .. 256+8l+7
    const uint2 p0 = lds64(coef_s + 32 * k + 8 * (lane / 16));
    const uint2 p1 = lds64(coef_s + 32 * k + 8 * (2 + lane / 16));
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const uint32_t w = b ? q11 : q01;
      const uint2 pc = b ? p1 : p0;
      const f2 c2{__uint_as_float(pc.x), __uint_as_float(pc.y)};
      const uint32_t ra = w * 32768u, rc = w * 128u;
      acc[4 * b + 0] = ffma2(f2{code_f<(3u << 15)>(ra, kC256), code_f<(3u << 17)>(ra, kC64)}, c2, acc[4 * b + 0]);
      acc[4 * b + 1] = ffma2(f2{code_f<(3u << 19)>(ra, kC16), code_f<(3u << 21)>(ra, kC4)}, c2, acc[4 * b + 1]);
      acc[4 * b + 2] = ffma2(f2{code_f<(3u << 15)>(rc, kC256), code_f<(3u << 17)>(rc, kC64)}, c2, acc[4 * b + 2]);
      acc[4 * b + 3] = ffma2(f2{code_f<(3u << 19)>(rc, kC16), code_f<(3u << 21)>(rc, kC4)}, c2, acc[4 * b + 3]);
    }
  };

  // Asynchronous form for the bf16 path: the records of a batch are copied to staging buffer
  // buf by cp.async (no registers held) while the warp streams bf16 columns and decodes the
  // previous batch; stage_ready waits for them and prepares the batch's coefficients. Lane k
  // fetches x of the batch's column k at issue, a batch ahead of its use, except in the masked
  // int4 kernel, which measured faster taking it at ready (its x mostly sits in shared memory).
  constexpr bool kXAtIssue = !FUSED || FMT == SPAX_FULL_BF16;
  float xn = 0.f;  // x of column `lane` of the batch in flight (0 for an invalid column)
  auto stage_issue = [&](int k0, int nb, int buf) {
    __syncwarp();  // every lane is done with what this buffer held
    const uint32_t dst = stage_s + kStage2Bytes * buf;
    for (int q = lane; q < nb * 9; q += 32) {
      const int k = q / 9, piece = q - 9 * k;
      const int col = max(colA(cg + CG * (k0 + k)), 0);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 16 * q),
                   "l"(p.approx + col * p.approx_col_stride + off_approx + 16 * piece)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    if (kXAtIssue && lane < nb) {
      const int i = cg + CG * (k0 + lane), col = colA(i);
      xn = col >= 0 ? xA(i, col) : 0.f;  // an invalid column contributes zero
    }
  };
  auto stage_ready = [&](int k0, int nb, int buf) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncwarp();
    if (lane < nb) {
      float xk = xn;
      if constexpr (!kXAtIssue) {
        const int i = cg + CG * (k0 + lane), col = colA(i);
        xk = col >= 0 ? xA(i, col) : 0.f;
      }
      const uint4 sm = lds128(stage_s + kStage2Bytes * buf + 144 * lane + 128);
      const uint32_t w[4] = {sm.x, sm.y, sm.z, sm.w};
      float c[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        c[g] = xk * __uint_as_float(w[g] << 16);
        sA[g] += c[g];
        bA[g] = fmaf(xk, __uint_as_float(w[g] & 0xFFFF0000u), bA[g]);
      }
      asm volatile("st.shared.v4.f32 [%0], {%1, %1, %2, %2};" ::"r"(coef_s + 32 * lane), "f"(c[0]),
                   "f"(c[1]));
      asm volatile("st.shared.v4.f32 [%0], {%1, %1, %2, %2};" ::"r"(coef_s + 32 * lane + 16),
                   "f"(c[2]), "f"(c[3]));
    }
    __syncwarp();
  };

  for (int ch = 0; ch < nchunks; ++ch) {
    const int ib0 = ch * kGemvMeta;
    const int nac = FUSED ? na : max(0, min(na - ib0, kGemvMeta));
    const int nfc = FUSED ? nf : max(0, min(nf - ib0, kGemvMeta));
    if constexpr (!FUSED) {
    if (ch > 0) {
      __syncthreads();  // every warp is done with the previous chunk's metadata
      if (!DENSE) {
        for (int i = tid; i < kGemvMeta; i += kGemvThreads) {
          const long long pos = split + (long long)S * (ib0 + i);
          if (i < nac) meta_col_a[i] = __ldcg(p.aidx + pos);
          if (i < nfc) meta_col_f[i] = __ldcg(p.fidx + pos);
        }
      }
    }
    // validate this chunk's columns (the dense GEMV generates them); an invalid one becomes -1.
    // (The fused kernel's lists come from its own selection: nothing to copy or check.)
    for (int i = tid; i < kGemvMeta; i += kGemvThreads) {
      if (i < nac && (unsigned)meta_col_a[i] >= (unsigned)p.d_in) {
        s_bad = 1;
        meta_col_a[i] = -1;
      }
      if (DENSE) {
        if (i < nfc) meta_col_f[i] = split + S * (ib0 + i);
      } else if (i < nfc && (unsigned)meta_col_f[i] >= (unsigned)p.d_in) {
        s_bad = 1;
        meta_col_f[i] = -1;
      }
    }
    __syncthreads();
    }
    if (!wrows) continue;
    const int nAw = nac > cg ? (nac - cg + CG - 1) / CG : 0;  // this warp's 2-bit columns
    const int nFw = nfc > cg ? (nfc - cg + CG - 1) / CG : 0;  // this warp's full columns

    if constexpr (FMT == SPAX_FULL_BF16) {
      // bf16 batches of U columns interleaved with 2-bit columns, so the dequant work of the
      // 2-bit tier runs while the bf16 loads are in flight
      // A last round of only 1-2 columns would cost the warp a memory round trip of its own; when
      // staging buffer 1 is idle (one 2-bit batch at most), those columns are fetched into it by
      // cp.async at once and added at the end. Only when the split's lists fit one chunk, so the
      // masked and the list-driven kernels take the same decision (the same order of sums).
      int ntail = 0;
      if (max(nf, na) <= kGemvMeta) {
        const int rounds = (nFw + U - 1) / U, last = nFw - U * (rounds - 1);
        if (rounds >= 2 && last <= 2 && nAw <= kBatch2) ntail = last;
      }
      const int nFr = nFw - ntail;  // columns through registers
      if (ntail) {
        __syncwarp();
        const uint32_t dst = stage_s + kStage2Bytes;  // buffer 1: 1 KB per column, 16 B per chunk
        for (int q = lane; q < 64 * ntail; q += 32) {
          const int t = q >> 6, c = q & 63;  // chunk c holds rows rb + 8c .. rb + 8c + 7
          const int col = max(colF(cg + CG * (nFr + t)), 0);
          if (rb + 8 * c < p.d_out)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 1024 * t + 16 * c),
                         "l"(p.full + col * p.full_col_stride + 2LL * rb + 16 * c)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
      }
      const int per_it = nFr > 0 ? (nAw * U + nFr - 1) / nFr : nAw;
      int ka = 0, kf = 0, sbeg = 0, send = 0, buf = 0;
      if (nAw > 0) stage_issue(0, min(kBatch2, nAw), 0);  // on its way before the first bf16 loads
      while (ka < nAw || kf < nFr) {
        const int nfb = max(0, min(U, nFr - kf));
        uint4 w0[U], w1[U];
        float xf[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = cg + CG * (kf + u);
          const int col = u < nfb ? colF(i) : -1;
          xf[u] = col >= 0 ? xF(i, col) : 0.f;
          const uint8_t* src = p.full + max(col, 0) * p.full_col_stride + off_full;
          w0[u] = (u < nfb && v0) ? ld_stream128(src) : make_uint4(0u, 0u, 0u, 0u);
          w1[u] = (u < nfb && v1) ? ld_stream128(src + 512) : make_uint4(0u, 0u, 0u, 0u);
        }
        int todo = (kf + nfb < nFr) ? min(per_it, nAw - ka) : nAw - ka;
        while (todo > 0) {
          if (ka == send) {  // the batch at ka is in flight: wait, then send the next one
            sbeg = ka;
            send = ka + min(kBatch2, nAw - ka);
            buf = (sbeg / kBatch2) & 1;
            stage_ready(sbeg, send - sbeg, buf);
            if (send < nAw) stage_issue(send, min(kBatch2, nAw - send), buf ^ 1);
          }
          const int n = min(todo, send - ka);
#pragma unroll 4
          for (int k = ka; k < ka + n; ++k) decode_approx(k - sbeg, buf);
          ka += n;
          todo -= n;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const f2 x2{xf[u], xf[u]};
          acc[0] = ffma2(bf16x2_to_f2(w0[u].x), x2, acc[0]);
          acc[1] = ffma2(bf16x2_to_f2(w0[u].y), x2, acc[1]);
          acc[2] = ffma2(bf16x2_to_f2(w0[u].z), x2, acc[2]);
          acc[3] = ffma2(bf16x2_to_f2(w0[u].w), x2, acc[3]);
          acc[4] = ffma2(bf16x2_to_f2(w1[u].x), x2, acc[4]);
          acc[5] = ffma2(bf16x2_to_f2(w1[u].y), x2, acc[5]);
          acc[6] = ffma2(bf16x2_to_f2(w1[u].z), x2, acc[6]);
          acc[7] = ffma2(bf16x2_to_f2(w1[u].w), x2, acc[7]);
        }
        kf += nfb;
      }
      if (ntail) {  // the tail columns, from buffer 1
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();
        for (int t = 0; t < ntail; ++t) {
          const int i = cg + CG * (nFr + t), col = colF(i);
          const f2 x2{col >= 0 ? xF(i, col) : 0.f, col >= 0 ? xF(i, col) : 0.f};
          const uint32_t src = stage_s + kStage2Bytes + 1024 * t + 16 * lane;
          const uint4 a = v0 ? lds128(src) : make_uint4(0u, 0u, 0u, 0u);
          const uint4 b = v1 ? lds128(src + 512) : make_uint4(0u, 0u, 0u, 0u);
          acc[0] = ffma2(bf16x2_to_f2(a.x), x2, acc[0]);
          acc[1] = ffma2(bf16x2_to_f2(a.y), x2, acc[1]);
          acc[2] = ffma2(bf16x2_to_f2(a.z), x2, acc[2]);
          acc[3] = ffma2(bf16x2_to_f2(a.w), x2, acc[3]);
          acc[4] = ffma2(bf16x2_to_f2(b.x), x2, acc[4]);
          acc[5] = ffma2(bf16x2_to_f2(b.y), x2, acc[5]);
          acc[6] = ffma2(bf16x2_to_f2(b.z), x2, acc[6]);
          acc[7] = ffma2(bf16x2_to_f2(b.w), x2, acc[7]);
        }
      }
    } else {
      // the 2-bit tier: batches double-buffered by cp.async, as in the bf16 path
      if (nAw > 0) stage_issue(0, min(kBatch2, nAw), 0);
      for (int ka = 0; ka < nAw; ka += kBatch2) {
        const int nb = min(kBatch2, nAw - ka), buf = (ka / kBatch2) & 1;
        stage_ready(ka, nb, buf);
        if (ka + kBatch2 < nAw) stage_issue(ka + kBatch2, min(kBatch2, nAw - ka - kBatch2), buf ^ 1);
#pragma unroll 2
        for (int k = 0; k < nb; ++k) decode_approx(k, buf);
      }
      // int4: 8 rows per word, nibble of row k at bits 4k, stored as u = q + 8. Shifts bring rows
      // (0,1), (2,3), (4,5), (6,7) to mantissa bits 15 and 19: values 256 + u and 16 + u. A staged
      // half-record is the warp's 256 bytes of nibbles followed by the record's 16 bytes of
      // scales (17 chunks of 16 B); batches of kBatch4 are double-buffered by cp.async in the
      // staging area, the next one in flight while the current one is decoded.
      auto stage4_issue = [&](int k0, int nb, int buf) {
        __syncwarp();  // every lane is done with what this buffer held
        const uint32_t dst = stage_s + kStage4Bytes * buf;
        for (int q = lane; q < nb * 17; q += 32) {
          const int k = q / 17, piece = q - 17 * k;
          const int col = max(colF(cg + CG * (k0 + k)), 0);
          const uint8_t* src = p.full + col * p.full_col_stride + (piece < 16 ? nib0 + 16 * piece : scl0);
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 16 * q), "l"(src)
                       : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        if (kXAtIssue && lane < nb) {
          const int i = cg + CG * (k0 + lane), col = colF(i);
          xn = col >= 0 ? xF(i, col) : 0.f;  // an invalid column contributes zero
        }
      };
      auto stage4_ready = [&](int k0, int nb, int buf) {
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();
        if (lane < nb) {
          float xk = xn;
          if constexpr (!kXAtIssue) {
            const int i = cg + CG * (k0 + lane), col = colF(i);
            xk = col >= 0 ? xF(i, col) : 0.f;
          }
          // this half's four group scales: bf16 scales [4*half4, 4*half4 + 4) of the record
          const uint2 sw = lds64(stage_s + kStage4Bytes * buf + 272 * lane + 256 + 8 * half4);
          const uint32_t w[4] = {sw.x << 16, sw.x & 0xFFFF0000u, sw.y << 16, sw.y & 0xFFFF0000u};
          float c[4];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            c[g] = xk * __uint_as_float(w[g]);
            s4[g] += c[g];
          }
          asm volatile("st.shared.v4.f32 [%0], {%1, %1, %2, %2};" ::"r"(coef_s + 32 * lane),
                       "f"(c[0]), "f"(c[1]));
          asm volatile("st.shared.v4.f32 [%0], {%1, %1, %2, %2};" ::"r"(coef_s + 32 * lane + 16),
                       "f"(c[2]), "f"(c[3]));
        }
        __syncwarp();
      };
      if (nFw > 0) stage4_issue(0, min(kBatch4, nFw), 0);
      for (int kf = 0; kf < nFw; kf += kBatch4) {
        const int nb = min(kBatch4, nFw - kf), buf = (kf / kBatch4) & 1;
        stage4_ready(kf, nb, buf);
        if (kf + kBatch4 < nFw) stage4_issue(kf + kBatch4, min(kBatch4, nFw - kf - kBatch4), buf ^ 1);
#pragma unroll 2
        for (int k = 0; k < nb; ++k) {
          const uint32_t rec = stage_s + kStage4Bytes * buf + 272 * k;
          const uint32_t n0 = lds32(rec + 4 * lane), n1 = lds32(rec + 128 + 4 * lane);
          const uint2 p0 = lds64(coef_s + 32 * k + 8 * (lane / 16));
          const uint2 p1 = lds64(coef_s + 32 * k + 8 * (2 + lane / 16));
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const uint32_t w = b ? n1 : n0;
            const uint2 pc = b ? p1 : p0;
            const f2 c2{__uint_as_float(pc.x), __uint_as_float(pc.y)};
            // shifts left by 15 and 7 as multiplies, right by 1 and 9 as the high words of
            // multiplies
            const uint32_t rA = w * 32768u, rB = w * 128u;
            const uint32_t rC = __umulhi(w, 0x80000000u), rD = __umulhi(w, 0x00800000u);
            acc[4 * b + 0] = ffma2(f2{code_f<(0xFu << 15)>(rA, kC256), code_f<(0xFu << 19)>(rA, kC16)}, c2, acc[4 * b + 0]);
            acc[4 * b + 1] = ffma2(f2{code_f<(0xFu << 15)>(rB, kC256), code_f<(0xFu << 19)>(rB, kC16)}, c2, acc[4 * b + 1]);
            acc[4 * b + 2] = ffma2(f2{code_f<(0xFu << 15)>(rC, kC256), code_f<(0xFu << 19)>(rC, kC16)}, c2, acc[4 * b + 2]);
            acc[4 * b + 3] = ffma2(f2{code_f<(0xFu << 15)>(rD, kC256), code_f<(0xFu << 19)>(rD, kC16)}, c2, acc[4 * b + 3]);
          }
        }
      }
    }
  }
  if (tid == 0 && s_bad) record_status(p.status, SPAX_ERR_INDEX);

  // warp totals of the per-group sums (xor butterfly: every lane ends with the same totals)
#pragma unroll
  for (int g = 0; g < 4; ++g) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      if constexpr (!DENSE) {
        sA[g] += __shfl_xor_sync(0xffffffffu, sA[g], o);
        bA[g] += __shfl_xor_sync(0xffffffffu, bA[g], o);
      }
      if constexpr (FMT == SPAX_FULL_INT4_G128) s4[g] += __shfl_xor_sync(0xffffffffu, s4[g], o);
    }
  }
  const int g0 = lane / 16;  // group of the lane's first 8 rows; the second chunk is group g0 + 2
  const float sumA0 = g0 ? sA[1] : sA[0], sumA1 = g0 ? sA[3] : sA[2];
  const float baseA0 = g0 ? bA[1] : bA[0], baseA1 = g0 ? bA[3] : bA[2];
  const float sum40 = g0 ? s4[1] : s4[0], sum41 = g0 ? s4[3] : s4[2];

  // ---- combine the warps' partial rows inside the CTA (fixed order) ----
  if (wrows) {
    // remove the mantissa constants: 2-bit rows 4i+{0,1,2,3} carry {256,64,16,4}*Σc, int4 even
    // rows (256+8)*Σc and odd rows (16+8)*Σc; add Σ x*min for the 2-bit tier
    float* slot = red + cg * kSlotFloats;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const float sa = b ? sumA1 : sumA0, ba = b ? baseA1 : baseA0, s4 = b ? sum41 : sum40;
      const float k0 = ba - 256.f * sa, k1 = ba - 64.f * sa, k2 = ba - 16.f * sa, k3 = ba - 4.f * sa;
      const float e = -264.f * s4, o = -24.f * s4;
      float4 lo, hi;
      lo.x = acc[4 * b + 0].x + k0 + e;
      lo.y = acc[4 * b + 0].y + k1 + o;
      lo.z = acc[4 * b + 1].x + k2 + e;
      lo.w = acc[4 * b + 1].y + k3 + o;
      hi.x = acc[4 * b + 2].x + k0 + e;
      hi.y = acc[4 * b + 2].y + k1 + o;
      hi.z = acc[4 * b + 3].x + k2 + e;
      hi.w = acc[4 * b + 3].y + k3 + o;
      float* dst = slot + red_row(512 * rg + 256 * b + 8 * lane);
      reinterpret_cast<float4*>(dst)[0] = lo;
      reinterpret_cast<float4*>(dst)[1] = hi;
    }
  }
  __syncthreads();
  // rows 4i..4i+3 of the tile: the column groups' slots summed in group order
  auto combined_rows = [&](int i) -> float4 {
    float4 v = reinterpret_cast<const float4*>(red + red_row(4 * i))[0];
#pragma unroll 3
    for (int c = 1; c < CG; ++c) {
      const float4 w = reinterpret_cast<const float4*>(red + c * kSlotFloats + red_row(4 * i))[0];
      v.x += w.x;
      v.y += w.y;
      v.z += w.z;
      v.w += w.w;
    }
    return v;
  };

  if (S == 1) {  // no split: the tile's rows are final
    for (int i = tid; i < rows_here / 4; i += kGemvThreads)
      reinterpret_cast<float4*>(p.y + r0)[i] = combined_rows(i);
    return;
  }

  // ---- split-K: publish this split's rows, then reduce one slice of the tile's rows ----
  // Each partial value travels with its ready flag in one 64-bit word (single-copy atomic), so
  // a reader that sees the flag sees the value: no fence, no counter, one trip through L2. The
  // S CTAs of a tile (all resident: the grid is one wave) each sum rows [4 g_lo, 4 g_hi) of the
  // tile over the S splits in split order (bit-reproducible) and clear the words they read, so
  // every completed call leaves the partial area at zero.
  unsigned long long* part = p.part + (size_t)split * p.d_out + r0;
  for (int i = tid; i < rows_here / 4; i += kGemvThreads) st_ll4(part + 4 * i, combined_rows(i));
  const int n4 = rows_here / 4;
  const int c4 = (n4 + S - 1) / S;
  const int g_lo = min(n4, split * c4), ng = min(n4, g_lo + c4) - g_lo;
  const int pairs = ng * S;  // (row group, source split) items, <= 2 per thread
  float4* sc = reinterpret_cast<float4*>(red);  // [S][c4]
  __syncthreads();  // the combine area is dead: reuse it as the gather scratch
  {
    const int q0 = tid, q1 = tid + kGemvThreads;
    const bool h0 = q0 < pairs, h1 = q1 < pairs;
    unsigned long long* a0 = h0 ? p.part + (size_t)(q0 / ng) * p.d_out + r0 + 4 * (g_lo + q0 % ng) : nullptr;
    unsigned long long* a1 = h1 ? p.part + (size_t)(q1 / ng) * p.d_out + r0 + 4 * (g_lo + q1 % ng) : nullptr;
    bool need0 = h0, need1 = h1;
    unsigned long long t0 = 0;
    for (int it = 0; need0 || need1; ++it) {
      float4 v;
      if (need0 && ld_ll4(a0, &v)) {
        sc[(q0 / ng) * c4 + q0 % ng] = v;
        clear_ll4(a0);
        need0 = false;
      }
      if (need1 && ld_ll4(a1, &v)) {
        sc[(q1 / ng) * c4 + q1 % ng] = v;
        clear_ll4(a1);
        need1 = false;
      }
      if ((need0 || need1) && (it & 15) == 15) {  // bounded: a missing split is a library bug
        const unsigned long long now = global_timer_ns();
        if (t0 == 0) t0 = now;
        else if (now - t0 > p.wait_ns) {
          record_status(p.status, SPAX_ERR_TIMEOUT);
          break;
        }
      }
    }
  }
  __syncthreads();
  for (int g = tid; g < ng; g += kGemvThreads) {
    float4 acc = sc[g];
    for (int q = 1; q < S; ++q) {
      const float4 v = sc[q * c4 + g];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    reinterpret_cast<float4*>(p.y + r0)[g_lo + g] = acc;
  }
}

// ------------------------------------------------------------------------------------------------

bool make_gemv_plan(int d_out, int d_in, int full_fmt, int sm_count, bool dense, GemvPlan* plan) {
  if (d_out < 128 || d_out % 128 != 0 || d_in < 1 || sm_count < 1) return false;
  if (full_fmt != SPAX_FULL_BF16 && full_fmt != SPAX_FULL_INT4_G128) return false;
  GemvPlan pl;
  pl.R = 2048;
  if (dense) {
    // Smallest row tile that still leaves >= 8 splits per tile: the dense stream gains from the
    // wider tiles of its compile-time instances.
    for (int r = 512; r <= 1024; r *= 2) {
      if ((d_out + r - 1) / r <= sm_count / 8) {
        pl.R = r;
        break;
      }
    }
  } else {
    // Smallest row tile whose one-wave grid keeps >= 85% of the SMs busy: fewer splits per tile
    // mean a shorter split-K exchange, and short tiles keep every CTA's share of a column small
    // (measured on the Llama-2-7B block: qkv 12 -> 6 splits and gate_up 13 -> 3 splits, 64.6 ->
    // 63.9 us per token-layer).
    for (int r = 512; r <= 1024; r *= 2) {
      const int t = (d_out + r - 1) / r;
      if (t <= sm_count && 100LL * t * (sm_count / t) >= 85LL * sm_count) {
        pl.R = r;
        break;
      }
    }
  }
  pl.T = (d_out + pl.R - 1) / pl.R;
  pl.S = sm_count / pl.T;
  if (pl.S < 1) pl.S = 1;
  if (pl.S > d_in) pl.S = d_in;
  if (pl.S > 256) pl.S = 256;  // keeps a CTA's reduction items within two per thread
  auto al = [](size_t v) { return (v + 255) & ~size_t(255); };
  pl.off_part = 0;
  pl.ws_bytes = pl.S > 1 ? al(size_t(pl.S) * d_out * 8) : 256;  // flagged 64-bit partials
  *plan = pl;
  return true;
}

template <int RGT, int FMT, bool DENSE, int FUSED>
static cudaError_t launch_one(const GemvParams& gp, const GemvPlan& pl, size_t smem,
                              cudaStream_t stream) {
  auto kern = tiered_gemv_kernel<RGT, FMT, DENSE, FUSED>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(pl.T, pl.S), dim3(kGemvThreads), smem, stream, gp);
}

template <int FMT, bool DENSE, int FUSED>
static cudaError_t launch_r(const GemvParams& gp, const GemvPlan& pl, size_t smem,
                            cudaStream_t stream) {
  if constexpr (DENSE) {
    if (pl.R == 512) return launch_one<1, FMT, DENSE, FUSED>(gp, pl, smem, stream);
    if (pl.R == 1024) return launch_one<2, FMT, DENSE, FUSED>(gp, pl, smem, stream);
    return launch_one<4, FMT, DENSE, FUSED>(gp, pl, smem, stream);
  } else {
    return launch_one<0, FMT, DENSE, FUSED>(gp, pl, smem, stream);
  }
}

static size_t gemv_smem_bytes() { return kGemvSmemBytes; }

// Shared memory of the masked GEMV: [metadata][staged lists][x, when it fits][reused area]. The
// reused area holds the selection's scratch, then the GEMV's combine and staging areas; x sits
// in it too (and the kernel stashes its split's x values) only when a separate x would not fit.
// *keys_bytes gets the separate x array's bytes (0: x in the reused area).
static size_t masked_gemv_layout(int d_in, size_t* keys_bytes) {
  const size_t meta = size_t(2) * kGemvMeta * 4;
  const size_t gemv = gemv_smem_bytes() - meta;  // combine + staging areas
  const size_t scratch = (sizeof(SelectSmem) + 15) / 16 * 16;
  const size_t alive = meta + select_list_bytes(d_in) + select_keys_bytes(d_in) +
                       (gemv > scratch ? gemv : scratch);
  if (alive <= kMaskedGemvSmemLimit) {
    *keys_bytes = select_keys_bytes(d_in);
    return alive;
  }
  const size_t sel = fused_select_bytes(d_in);
  *keys_bytes = 0;
  return meta + select_list_bytes(d_in) + (gemv > sel ? gemv : sel);
}

size_t masked_gemv_smem_bytes(const GemvPlan& /*pl: every tile height takes the same*/, int d_in) {
  size_t kb;
  return masked_gemv_layout(d_in, &kb);
}

static GemvParams make_params(const GemvLaunch& a, const GemvPlan& pl) {
  GemvParams gp = {};
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  gp.full = static_cast<const uint8_t*>(a.full);
  gp.approx = static_cast<const uint8_t*>(a.approx);
  gp.x = a.x;
  gp.fidx = a.full_idx;
  gp.aidx = a.approx_idx;
  gp.counts = a.counts;
  gp.y = a.y;
  gp.part = reinterpret_cast<unsigned long long*>(ws + pl.off_part);
  gp.status = a.status;
  gp.full_col_stride = a.full_fmt == SPAX_FULL_BF16 ? 2LL * a.d_out
                                                    : (long long)((a.d_out + 1023) / 1024) * 528;
  gp.approx_col_stride = (long long)((a.d_out + 511) / 512) * 144;
  gp.d_out = a.d_out;
  gp.d_in = a.d_in;
  gp.S = pl.S;
  gp.RG = pl.R / 512;
  gp.list_bytes = 0;
  gp.keys_bytes = 0;
  gp.wait_ns = a.wait_ns ? a.wait_ns : kWaitLimitNs;
  return gp;
}

cudaError_t launch_gemv(const GemvLaunch& a, const GemvPlan& pl, cudaStream_t stream) {
  const GemvParams gp = make_params(a, pl);
  const size_t smem = gemv_smem_bytes();
  GemvPlan grid = pl;  // the launched grid: every split, or (a failure-detection test) fewer
  grid.S = pl.S - a.drop_splits;
  if (grid.S < 1) return cudaErrorInvalidValue;
  if (a.dense) return launch_r<SPAX_FULL_BF16, true, 0>(gp, grid, smem, stream);
  if (a.full_fmt == SPAX_FULL_BF16) return launch_r<SPAX_FULL_BF16, false, 0>(gp, grid, smem, stream);
  return launch_r<SPAX_FULL_INT4_G128, false, 0>(gp, grid, smem, stream);
}

// The masked instance of a FUSED value (source | kFusedScaled).
template <int FMT>
static cudaError_t launch_src(const GemvParams& gp, const GemvPlan& pl, size_t smem, int src,
                              cudaStream_t stream) {
  switch (src) {
    case kFusedSwiglu: return launch_r<FMT, false, kFusedSwiglu>(gp, pl, smem, stream);
    case kFusedScored: return launch_r<FMT, false, kFusedScored>(gp, pl, smem, stream);
    case kFusedX | kFusedScaled: return launch_r<FMT, false, kFusedX | kFusedScaled>(gp, pl, smem, stream);
    case kFusedSwiglu | kFusedScaled:
      return launch_r<FMT, false, kFusedSwiglu | kFusedScaled>(gp, pl, smem, stream);
    case kFusedScored | kFusedScaled:
      return launch_r<FMT, false, kFusedScored | kFusedScaled>(gp, pl, smem, stream);
    default: return launch_r<FMT, false, kFusedX>(gp, pl, smem, stream);
  }
}

cudaError_t launch_masked_gemv(const GemvLaunch& a, const spax_mask_params& prm, bool swiglu,
                               float* x_out, const float* norms, uint8_t* tier, int32_t* full_idx,
                               int32_t* approx_idx, int32_t* counts, const GemvPlan& pl,
                               cudaStream_t stream) {
  GemvParams gp = make_params(a, pl);
  gp.prm = prm;
  gp.x_out = swiglu ? x_out : nullptr;
  gp.norms = swiglu ? nullptr : norms;
  gp.tier_out = tier;
  gp.fidx_out = full_idx;
  gp.aidx_out = approx_idx;
  gp.counts_out = counts;
  gp.list_bytes = (int)select_list_bytes(a.d_in);
  size_t kb;
  const size_t smem = masked_gemv_layout(a.d_in, &kb);
  gp.keys_bytes = (int)kb;
  // A SwiGLU call whose product finds every x in shared memory (x kept alive, or each split's
  // positions within the stash for any count) runs the plain instance, which forms x in its
  // fetch: the layer's launches then share one image (warm in the instruction caches).
  const int per_split = (a.d_in + pl.S - 1) / pl.S;
  int src = kFusedX;
  if (swiglu && (kb != 0 || per_split <= kGemvMeta))
    gp.fetch_swiglu = 1;
  else if (swiglu)
    src = kFusedSwiglu;
  else if (norms)
    src = kFusedScored;
  if (prm.mode == SPAX_MASK_TOPK_SCALED) src |= kFusedScaled;
  if (a.full_fmt == SPAX_FULL_BF16) return launch_src<SPAX_FULL_BF16>(gp, pl, smem, src, stream);
  return launch_src<SPAX_FULL_INT4_G128>(gp, pl, smem, src, stream);
}

}  // namespace spax
