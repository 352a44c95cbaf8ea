/*
 * spax_oracle.c — plain, slow, obviously correct CPU reference of the three-tier decode GEMV.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call this file; only
 * the test suite, the smoke check and the CPU-baseline leg of the benchmark use it. It shares no
 * code, header, table or helper with the CUDA library: every format and rule below is written
 * out here again from its definition.
 *
 * Sources (page title, section):
 *   [SpAx]  "SpAx: Activation Sparsity with Weight Approximation for Faster LLM Decoding on
 *           Offloaded Weights", Abstract: skip the columns whose activations are closest to zero,
 *           read approximate (compressed) weights for smaller magnitudes, original weights for
 *           the largest.
 *   [ER]    eigenradar commentary on SpAx, "The route outside GPU memory": a column is in the
 *           original, two-bit approximate or unread tier by activation magnitude; bytes moved per
 *           token are the unit of cost.
 *   [TKG]   "TopK-Guided: Adaptive, Budget-Aware Activation Sparsity for Efficient LLM
 *           Inference": Abstract and §1 (threshold rule of TEAL, fixed-count TopK rule of WINA),
 *           §2.1 (natural sparsity from the calibrated threshold clipped to target ±δ, then TopK),
 *           §2.2 (block budgets: less sparsity for sensitive blocks, λ, clamp [0.05, 0.95]).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - rank order: larger |x| first, equal |x| broken by the lower column index first;
 *   - guided bands in integer basis points: m = min(max(n, ceil((s-δ)d)), floor((s+δ)d)) with
 *     the upper end capped at d, and the three-tier split applies the clip at both boundaries;
 *   - quantile rank min(floor(s*M + 1/2), M-1) of the ascending pooled |x|;
 *   - 2-bit asymmetric min/max quantiser and int4 symmetric absmax quantiser per 128-row group,
 *     fp32 arithmetic with round-to-nearest-even, codes taken against the stored bf16 scale/min;
 *   - budget rule s_b = clamp(s(1 - λ(σ_b/σ̄ - 1)) + c, lo, hi) with c restoring the mean.
 *
 * Floating point: the quantiser is evaluated in IEEE fp32 (this file is compiled without FMA
 * contraction); products are accumulated in fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_OK 0
#define OR_ERR_ARG 1
#define OR_ERR_SHAPE 2
#define OR_ERR_NONFINITE 5

#define OR_FULL_BF16 0
#define OR_FULL_INT4 1

#define OR_MODE_THRESHOLD 0
#define OR_MODE_TOPK 1
#define OR_MODE_GUIDED 2

/* ------------------------------------------------------------------ bf16 <-> fp32 ---------- */

static float f32_from_bits(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return f;
}
static uint32_t bits_from_f32(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

/* bf16 value -> fp32 (exact: bf16 is the top half of an fp32). */
float oracle_bf16_to_f32(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/*
 * fp32 -> bf16, round to nearest, ties to even, written from the definition: keep the top 16
 * bits, and round up when the dropped 16 bits exceed half an ulp, or equal half an ulp and the
 * kept part is odd. NaN stays a quiet NaN.
 */
uint16_t oracle_f32_to_bf16(float f) {
  uint32_t u = bits_from_f32(f);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0) {
    return (uint16_t)((u >> 16) | 0x0040u);
  }
  uint32_t kept = u >> 16;
  uint32_t dropped = u & 0xFFFFu;
  if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1u;
  return (uint16_t)kept;
}

/* ------------------------------------------------------------------ tier rule --------------- */

typedef struct {
  float key;
  int32_t j;
} keyed_t;

/* "a before b" iff |x_a| > |x_b|, or equal magnitudes and a has the lower column index. */
static int cmp_rank(const void* pa, const void* pb) {
  const keyed_t* a = (const keyed_t*)pa;
  const keyed_t* b = (const keyed_t*)pb;
  if (a->key > b->key) return -1;
  if (a->key < b->key) return 1;
  return (a->j < b->j) ? -1 : (a->j > b->j);
}

/* Clip a natural count n into the guided band around target s (basis points), TKG §2.1. */
static int64_t guided_clip(int64_t n, int64_t d, int64_t s_bp, int64_t delta_bp) {
  int64_t lo_num = (s_bp - delta_bp) * d;
  int64_t lo = lo_num <= 0 ? 0 : (lo_num + 9999) / 10000; /* ceil */
  int64_t hi = (s_bp + delta_bp) * d / 10000;             /* floor */
  if (hi > d) hi = d;
  int64_t m = n < lo ? lo : n;
  if (m > hi) m = hi;
  return m;
}

/*
 * oracle_tiers: the tier of every column of one token and the ascending compacted lists.
 *   mode THRESHOLD: skip |x|<t_skip, approx t_skip<=|x|<t_full, else full   (TKG Abstract, §1)
 *   mode TOPK:      rank r(j) by the order above; full r<k_full, approx next k_approx (TKG §1)
 *   mode GUIDED:    n1=#{|x|<t_skip}, n2=#{|x|<t_full}; m1, m2 = band clips; m2 = max(m2, m1);
 *                   then TOPK with k_full = d - m2, k_approx = m2 - m1               (TKG §2.1)
 * counts[4] = {n_full, n_approx, n1, n2} (n1 = n2 = 0 for TOPK). Returns OR_ERR_NONFINITE (all
 * tiers 0, counts 0) if some x_j is NaN or Inf.
 */
int oracle_tiers(const float* x, int d, int mode, float t_skip, float t_full, int k_full,
                 int k_approx, int s_skip_bp, int s_below_full_bp, int delta_bp, uint8_t* tier,
                 int32_t* full_idx, int32_t* approx_idx, int32_t* counts) {
  if (d < 0 || !x || !tier || !full_idx || !approx_idx || !counts) return OR_ERR_ARG;
  for (int i = 0; i < 4; ++i) counts[i] = 0;
  for (int j = 0; j < d; ++j) {
    if (!isfinite(x[j])) {
      memset(tier, 0, (size_t)d);
      return OR_ERR_NONFINITE;
    }
  }
  int64_t n1 = 0, n2 = 0;
  if (mode == OR_MODE_THRESHOLD || mode == OR_MODE_GUIDED) {
    for (int j = 0; j < d; ++j) {
      float a = fabsf(x[j]);
      if (a < t_skip) ++n1;
      if (a < t_full) ++n2;
    }
  }
  if (mode == OR_MODE_THRESHOLD) {
    for (int j = 0; j < d; ++j) {
      float a = fabsf(x[j]);
      tier[j] = a < t_skip ? 0 : (a < t_full ? 1 : 2);
    }
  } else if (mode == OR_MODE_TOPK || mode == OR_MODE_GUIDED) {
    int64_t kf, ka;
    if (mode == OR_MODE_TOPK) {
      kf = k_full;
      ka = k_approx;
    } else {
      int64_t m1 = guided_clip(n1, d, s_skip_bp, delta_bp);
      int64_t m2 = guided_clip(n2, d, s_below_full_bp, delta_bp);
      if (m2 < m1) m2 = m1;
      kf = d - m2;
      ka = m2 - m1;
    }
    if (kf < 0 || ka < 0 || kf + ka > d) return OR_ERR_ARG;
    keyed_t* ord = (keyed_t*)malloc(sizeof(keyed_t) * (size_t)(d > 0 ? d : 1));
    if (!ord) return OR_ERR_ARG;
    for (int j = 0; j < d; ++j) {
      ord[j].key = fabsf(x[j]);
      ord[j].j = j;
    }
    qsort(ord, (size_t)d, sizeof(keyed_t), cmp_rank);
    for (int r = 0; r < d; ++r) {
      int j = ord[r].j;
      tier[j] = r < kf ? 2 : (r < kf + ka ? 1 : 0);
    }
    free(ord);
  } else {
    return OR_ERR_ARG;
  }
  int nf = 0, na = 0;
  for (int j = 0; j < d; ++j) {
    if (tier[j] == 2) full_idx[nf++] = j;
    if (tier[j] == 1) approx_idx[na++] = j;
  }
  counts[0] = nf;
  counts[1] = na;
  if (mode != OR_MODE_TOPK) {
    counts[2] = (int32_t)n1;
    counts[3] = (int32_t)n2;
  }
  return OR_OK;
}

/* ------------------------------------------------------------------ quantisers -------------- */

/*
 * 2-bit asymmetric quantiser of one 128-row group (values w[0..n) as bf16 bits), fp32:
 *   mn, mx = min, max (a zero extreme counts as +0); min_b = bf16(mn) (exact, mn is a bf16
 *   value); scale_b = bf16_rne((mx-mn)/3);
 *   q = clamp(rint_even((w - min_b) / scale_b), 0, 3), or 0 when scale_b == 0.
 * Dequantised value: min_b + q * scale_b.
 */
void oracle_quant2_group(const uint16_t* w, int n, uint8_t* q, uint16_t* scale_b,
                         uint16_t* min_b) {
  float mn = oracle_bf16_to_f32(w[0]), mx = mn;
  for (int i = 1; i < n; ++i) {
    float v = oracle_bf16_to_f32(w[i]);
    if (v < mn) mn = v;
    if (v > mx) mx = v;
  }
  /* a zero extreme is taken as +0 (adding +0 maps -0 to +0 and leaves every other value) */
  volatile float mn0 = mn + 0.0f, mx0 = mx + 0.0f;
  mn = mn0;
  mx = mx0;
  volatile float range = mx - mn; /* volatile: keep each fp32 step rounded on its own */
  volatile float third = range / 3.0f;
  uint16_t sb = oracle_f32_to_bf16(third);
  uint16_t mb = oracle_f32_to_bf16(mn);
  float s = oracle_bf16_to_f32(sb), m = oracle_bf16_to_f32(mb);
  for (int i = 0; i < n; ++i) {
    int code = 0;
    if (s != 0.0f) {
      volatile float diff = oracle_bf16_to_f32(w[i]) - m;
      volatile float ratio = diff / s;
      float r = nearbyintf(ratio); /* default rounding mode: to nearest, ties to even */
      code = r < 0.0f ? 0 : (r > 3.0f ? 3 : (int)r);
    }
    q[i] = (uint8_t)code;
  }
  *scale_b = sb;
  *min_b = mb;
}

/*
 * int4 symmetric quantiser of one 128-row group, fp32: scale_b = bf16_rne(max|w| / 7);
 * q = clamp(rint_even(w / scale_b), -8, 7), or 0 when scale_b == 0. Value: q * scale_b.
 */
void oracle_quant4_group(const uint16_t* w, int n, int8_t* q, uint16_t* scale_b) {
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) {
    float v = fabsf(oracle_bf16_to_f32(w[i]));
    if (v > amax) amax = v;
  }
  volatile float sev = amax / 7.0f;
  uint16_t sb = oracle_f32_to_bf16(sev);
  float s = oracle_bf16_to_f32(sb);
  for (int i = 0; i < n; ++i) {
    int code = 0;
    if (s != 0.0f) {
      volatile float ratio = oracle_bf16_to_f32(w[i]) / s;
      float r = nearbyintf(ratio);
      code = r < -8.0f ? -8 : (r > 7.0f ? 7 : (int)r);
    }
    q[i] = (int8_t)code;
  }
  *scale_b = sb;
}

/* ------------------------------------------------------------------ packed layout ----------- */
/*
 * The packed layout (the interface both sides implement from the same written definition):
 *   full bf16:  W^T [d_in][d_out] bf16.
 *   full int4:  per column, ceil(d_out/1024) records of 528 B: 512 B of nibbles (row 2b low,
 *               2b+1 high nibble of byte b, nibble = q + 8) then 8 bf16 scales.
 *   approx:     per column, ceil(d_out/512) records of 144 B: 128 B of 2-bit codes (row r of
 *               the record at bits 2(r%4) of byte r/4) then 4 uint32 words (scale | min<<16).
 *   Padding rows: 2-bit code 0, scale = min = 0; int4 nibble 8, scale 0.
 */
static int64_t n_rec2(int d_out) { return (d_out + 511) / 512; }
static int64_t n_rec4(int d_out) { return (d_out + 1023) / 1024; }

int64_t oracle_full_col_bytes(int d_out, int fmt) {
  return fmt == OR_FULL_BF16 ? 2 * (int64_t)d_out : n_rec4(d_out) * 528;
}
int64_t oracle_approx_col_bytes(int d_out) { return n_rec2(d_out) * 144; }

static void put_u16(uint8_t* p, uint16_t v) {
  p[0] = (uint8_t)(v & 0xFF);
  p[1] = (uint8_t)(v >> 8);
}
static uint16_t get_u16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/*
 * Pack column j of the row-major bf16 matrix W [d_out][d_in] into its full-pool column
 * (full_col, oracle_full_col_bytes bytes) and approx-pool column (approx_col).
 */
int oracle_pack_column(const uint16_t* W, int d_out, int d_in, int fmt, int j, uint8_t* full_col,
                       uint8_t* approx_col) {
  if (d_out < 128 || d_out % 128 != 0 || d_in < 1 || j < 0 || j >= d_in) return OR_ERR_SHAPE;
  if (fmt != OR_FULL_BF16 && fmt != OR_FULL_INT4) return OR_ERR_ARG;
  uint16_t grp[128];
  uint8_t q2[128];
  int8_t q4[128];
  /* approx pool */
  memset(approx_col, 0, (size_t)oracle_approx_col_bytes(d_out));
  for (int g = 0; g < d_out / 128; ++g) {
    for (int i = 0; i < 128; ++i) grp[i] = W[(int64_t)(g * 128 + i) * d_in + j];
    uint16_t sb, mb;
    oracle_quant2_group(grp, 128, q2, &sb, &mb);
    int rec = g / 4, gi = g % 4;
    uint8_t* r = approx_col + (int64_t)rec * 144;
    for (int i = 0; i < 128; ++i) {
      int row_in_rec = gi * 128 + i;
      r[row_in_rec / 4] |= (uint8_t)(q2[i] << (2 * (row_in_rec % 4)));
    }
    put_u16(r + 128 + 4 * gi, sb);
    put_u16(r + 128 + 4 * gi + 2, mb);
  }
  /* full pool */
  if (fmt == OR_FULL_BF16) {
    for (int r = 0; r < d_out; ++r) put_u16(full_col + 2 * r, W[(int64_t)r * d_in + j]);
  } else {
    int64_t nb = n_rec4(d_out);
    memset(full_col, 0x88, (size_t)(nb * 528)); /* padding nibbles: q = 0 */
    for (int64_t b = 0; b < nb; ++b) memset(full_col + b * 528 + 512, 0, 16);
    for (int g = 0; g < d_out / 128; ++g) {
      for (int i = 0; i < 128; ++i) grp[i] = W[(int64_t)(g * 128 + i) * d_in + j];
      uint16_t sb;
      oracle_quant4_group(grp, 128, q4, &sb);
      int rec = g / 8, gi = g % 8;
      uint8_t* r = full_col + (int64_t)rec * 528;
      for (int i = 0; i < 128; ++i) {
        int row_in_rec = gi * 128 + i;
        uint8_t u = (uint8_t)(q4[i] + 8);
        uint8_t* byte = r + row_in_rec / 2;
        if (row_in_rec % 2 == 0)
          *byte = (uint8_t)((*byte & 0xF0) | u);
        else
          *byte = (uint8_t)((*byte & 0x0F) | (u << 4));
      }
      put_u16(r + 512 + 2 * gi, sb);
    }
  }
  return OR_OK;
}

/* Pack every column: full pool [d_in] columns back to back, approx pool likewise. */
int oracle_pack(const uint16_t* W, int d_out, int d_in, int fmt, uint8_t* full, uint8_t* approx) {
  int64_t fcb = oracle_full_col_bytes(d_out, fmt), acb = oracle_approx_col_bytes(d_out);
  for (int j = 0; j < d_in; ++j) {
    int rc = oracle_pack_column(W, d_out, d_in, fmt, j, full + fcb * j, approx + acb * j);
    if (rc) return rc;
  }
  return OR_OK;
}

/* Dequantised value of row r of a packed full-pool column. */
double oracle_full_value(const uint8_t* full_col, int fmt, int r) {
  if (fmt == OR_FULL_BF16) return (double)oracle_bf16_to_f32(get_u16(full_col + 2 * r));
  const uint8_t* rec = full_col + (int64_t)(r / 1024) * 528;
  int rr = r % 1024;
  uint8_t byte = rec[rr / 2];
  int u = (rr % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
  float s = oracle_bf16_to_f32(get_u16(rec + 512 + 2 * (rr / 128)));
  return (double)(u - 8) * (double)s;
}

/* Dequantised value of row r of a packed approx-pool column: min + q * scale. */
double oracle_approx_value(const uint8_t* approx_col, int r) {
  const uint8_t* rec = approx_col + (int64_t)(r / 512) * 144;
  int rr = r % 512;
  int q = (rec[rr / 4] >> (2 * (rr % 4))) & 3;
  int g = rr / 128;
  float s = oracle_bf16_to_f32(get_u16(rec + 128 + 4 * g));
  float m = oracle_bf16_to_f32(get_u16(rec + 128 + 4 * g + 2));
  return (double)m + (double)q * (double)s;
}

/* ------------------------------------------------------------------ products --------------- */

/*
 * Tiered product of one token, fp64 accumulation [SpAx Abstract; ER]:
 *   y_r = Σ_{j: tier 2} x_j * full(r, j) + Σ_{j: tier 1} x_j * approx(r, j).
 * rows == NULL: all d_out rows into y[d_out]; else the n_rows listed rows into y[n_rows].
 */
int oracle_tiered_gemv(const uint8_t* full, const uint8_t* approx, int fmt, int d_out, int d_in,
                       const float* x, const uint8_t* tier, const int32_t* rows, int n_rows,
                       double* y) {
  if (d_out < 128 || d_out % 128 != 0 || d_in < 1) return OR_ERR_SHAPE;
  int64_t fcb = oracle_full_col_bytes(d_out, fmt), acb = oracle_approx_col_bytes(d_out);
  int ny = rows ? n_rows : d_out;
  /* Outputs in chunks of 256 rows, each chunk summing its columns in ascending j. The chunks are
     independent: the multi-core build (OpenMP) hands them to threads; every y[i] is the same
     sum in the same order either way. */
#pragma omp parallel for schedule(dynamic, 1)
  for (int c0 = 0; c0 < ny; c0 += 256) {
    int c1 = ny - c0 < 256 ? ny : c0 + 256;
    for (int i = c0; i < c1; ++i) y[i] = 0.0;
    for (int j = 0; j < d_in; ++j) {
      if (tier[j] == 0) continue;
      double xj = (double)x[j];
      for (int i = c0; i < c1; ++i) {
        int r = rows ? rows[i] : i;
        double w = tier[j] == 2 ? oracle_full_value(full + fcb * j, fmt, r)
                                : oracle_approx_value(approx + acb * j, r);
        y[i] += xj * w;
      }
    }
  }
  return OR_OK;
}

/* Dense product y = W x from the row-major bf16 matrix, fp64 accumulation. */
int oracle_dense_gemv(const uint16_t* W, int d_out, int d_in, const float* x, const int32_t* rows,
                      int n_rows, double* y) {
  int ny = rows ? n_rows : d_out;
  for (int i = 0; i < ny; ++i) {
    int r = rows ? rows[i] : i;
    double acc = 0.0;
    for (int j = 0; j < d_in; ++j)
      acc += (double)x[j] * (double)oracle_bf16_to_f32(W[(int64_t)r * d_in + j]);
    y[i] = acc;
  }
  return OR_OK;
}

/*
 * Column norms for the WINA score [TKG §C.1: the per-element score of a column is the
 * activation's magnitude times the column's norm]: norm_j = (float) sqrt(Σ_r W[r][j]^2), the
 * squares (exact in fp64) summed in fp64 in row order, sqrt correctly rounded, one rounding to
 * fp32.
 */
int oracle_column_norms(const uint16_t* W, int d_out, int d_in, float* norms) {
  if (d_out < 1 || d_in < 1) return OR_ERR_SHAPE;
  for (int j = 0; j < d_in; ++j) {
    double acc = 0.0;
    for (int r = 0; r < d_out; ++r) {
      double w = (double)oracle_bf16_to_f32(W[(int64_t)r * d_in + j]);
      acc += w * w;
    }
    norms[j] = (float)sqrt(acc);
  }
  return OR_OK;
}

/* Threads the products use: 1 in the plain build, the OpenMP team size in the multi-core one. */
int oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------ calibration ----------- */

static int cmp_float_asc(const void* pa, const void* pb) {
  float a = *(const float*)pa, b = *(const float*)pb;
  return (a > b) - (a < b);
}

/*
 * Calibrated thresholds [TKG §2.1 "calibrated threshold", §2.2]: pool the M values |x| of the
 * calibration tokens, sort ascending into v, and take t(s) = v[min(floor(s*M + 1/2), M-1)] for
 * s = s_skip_bp/1e4 (t_skip) and s = s_below_full_bp/1e4 (t_full), integer index arithmetic.
 */
int oracle_calibrate(const float* X, int64_t M, int s_skip_bp, int s_below_full_bp,
                     float* t_out) {
  if (M < 1) return OR_ERR_ARG;
  float* v = (float*)malloc(sizeof(float) * (size_t)M);
  if (!v) return OR_ERR_ARG;
  for (int64_t i = 0; i < M; ++i) {
    if (!isfinite(X[i])) {
      free(v);
      return OR_ERR_NONFINITE;
    }
    v[i] = fabsf(X[i]);
  }
  qsort(v, (size_t)M, sizeof(float), cmp_float_asc);
  int bps[2] = {s_skip_bp, s_below_full_bp};
  for (int k = 0; k < 2; ++k) {
    int64_t idx = ((int64_t)bps[k] * M + 5000) / 10000;
    if (idx > M - 1) idx = M - 1;
    t_out[k] = v[idx];
  }
  free(v);
  return OR_OK;
}

/* ------------------------------------------------------------------ block budgets --------- */

static double clampd(double v, double lo, double hi) { return v < lo ? lo : (v > hi ? hi : v); }

static double mean_clamped(const double* a, int n, double c, double lo, double hi) {
  double s = 0.0;
  for (int b = 0; b < n; ++b) s += clampd(a[b] + c, lo, hi);
  return s / n;
}

static int cmp_double_asc(const void* pa, const void* pb) {
  double a = *(const double*)pa, b = *(const double*)pb;
  return (a > b) - (a < b);
}

/*
 * Block budgets [TKG §2.2]: a_b = s(1 - λ(σ_b/σ̄ - 1)); s_b = clamp(a_b + c, lo, hi) with the
 * shift c solving mean_b s_b = s. The mean is a continuous, non-decreasing, piecewise-linear
 * function of c with breakpoints lo - a_b and hi - a_b, so c is found exactly: locate the two
 * consecutive breakpoints whose values bracket s and interpolate on that linear piece.
 */
int oracle_block_budgets(const double* sens, int n, double s, double lambda, double lo, double hi,
                         double* out) {
  if (n < 1 || !(lo <= s && s <= hi) || lambda < 0.0) return OR_ERR_ARG;
  double sbar = 0.0;
  for (int b = 0; b < n; ++b) sbar += sens[b];
  sbar /= n;
  double* a = (double*)malloc(sizeof(double) * (size_t)n);
  double* bp = (double*)malloc(sizeof(double) * (size_t)(2 * n));
  for (int b = 0; b < n; ++b) {
    a[b] = s * (1.0 - lambda * (sens[b] / sbar - 1.0));
    bp[2 * b] = lo - a[b];
    bp[2 * b + 1] = hi - a[b];
  }
  qsort(bp, (size_t)(2 * n), sizeof(double), cmp_double_asc);
  double c = 0.0;
  if (mean_clamped(a, n, 0.0, lo, hi) != s) {
    /* mean at bp[0] is lo, at bp[2n-1] is hi; find k with f(bp[k]) <= s <= f(bp[k+1]). */
    int found = 0;
    for (int k = 0; k + 1 < 2 * n; ++k) {
      double f0 = mean_clamped(a, n, bp[k], lo, hi), f1 = mean_clamped(a, n, bp[k + 1], lo, hi);
      if (f0 <= s && s <= f1) {
        c = (f1 == f0) ? bp[k] : bp[k] + (s - f0) * (bp[k + 1] - bp[k]) / (f1 - f0);
        found = 1;
        break;
      }
    }
    if (!found) c = (s <= lo) ? bp[0] : bp[2 * n - 1];
  }
  for (int b = 0; b < n; ++b) out[b] = clampd(a[b] + c, lo, hi);
  free(a);
  free(bp);
  return OR_OK;
}

/* ------------------------------------------------------------------ byte account ---------- */

/*
 * Weight bytes of one tiered product [ER "bytes moved for each generated token"]:
 * n_full columns at 2*d_out bytes (bf16) or d_out/2 + 2*(d_out/128) bytes (int4 codes + bf16
 * scales), plus n_approx columns at d_out/4 bytes of codes + 4*(d_out/128) bytes of scale/min.
 */
uint64_t oracle_weight_bytes(int d_out, int fmt, int64_t n_full, int64_t n_approx) {
  uint64_t groups = (uint64_t)d_out / 128;
  uint64_t per_full = fmt == OR_FULL_BF16 ? 2ull * d_out : (uint64_t)d_out / 2 + 2 * groups;
  uint64_t per_approx = (uint64_t)d_out / 4 + 4 * groups;
  return (uint64_t)n_full * per_full + (uint64_t)n_approx * per_approx;
}
