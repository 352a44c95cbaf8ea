/*
 * spax.h — C ABI of libspax.so: three-tier, activation-sparse decode GEMV on B200 (sm_100a).
 *
 * What the library computes (one token, batch-one decode, one projection y = W·x):
 *   Every weight column j of W (d_out × d_in) is put in one of three tiers by the magnitude of
 *   the activation x_j: skipped (|x_j| closest to zero), read as a 2-bit approximation (smaller
 *   |x_j|), or read in its original format (largest |x_j|).
 *   Source: "SpAx: Activation Sparsity with Weight Approximation for Faster LLM Decoding on
 *   Offloaded Weights" (arXiv 2610.02598), Abstract; eigenradar commentary on SpAx, section
 *   "The route outside GPU memory" (original / two-bit approximate / unread tier per column).
 *   The tier rules (threshold, TopK, TopK-Guided ±δ clip) follow "TopK-Guided: Adaptive,
 *   Budget-Aware Activation Sparsity for Efficient LLM Inference" (arXiv 2610.01763),
 *   Abstract, §1 and §2.1; the block budgets follow its §2.2.
 *
 * Conventions shared by every entry point
 *   - Pointers named d_* (and every tensor argument of a device call) are DEVICE pointers;
 *     pointers named h_* are HOST pointers. The caller owns all memory; the library never
 *     allocates and keeps no state except a per-device cache of the SM count.
 *   - Device calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the
 *     legacy default stream) and never synchronise the host. Kernels are launched with the
 *     programmatic-dependent-launch attribute, so consecutive spax calls on one stream (and in
 *     a captured CUDA graph) overlap launch latency; every kernel waits for its predecessor
 *     before touching global memory.
 *   - The returned spax_status reports argument/shape errors (nothing is launched) and launch
 *     errors (SPAX_ERR_CUDA). Data-dependent errors found on the device (non-finite input,
 *     malformed index lists, a pipeline wait that ran out) are written to *d_status (an int32
 *     on the device, may be NULL) as a spax_status value; the caller reads it after a sync.
 *     A kernel never clears *d_status; the caller zeroes it.
 *   - Every pointer is aligned for its element type (4 bytes for float and int32, 8 for
 *     double). Entry points that need more (16-byte pools and outputs, 256-byte workspaces)
 *     say so and return SPAX_ERR_ARG when it does not hold.
 *   - Tier codes: 0 = skip, 1 = approximate (2-bit), 2 = full (original format).
 *   - Compacted column lists are in ascending column order.
 *
 * Packed weight layout (produced by spax_pack_weights, read by spax_tiered_gemv)
 *   The dense matrix W arrives row-major [d_out][d_in] bf16 (the nn.Linear layout). Packing
 *   makes every column contiguous, so a selected column is one contiguous run in HBM.
 *   d_out must be a multiple of 128 (the quantisation group).
 *   full pool, SPAX_FULL_BF16: W^T as bf16 [d_in][d_out]; column stride 2*d_out bytes.
 *   full pool, SPAX_FULL_INT4_G128: per column, ceil(d_out/1024) records of 528 bytes:
 *       512 bytes of 4-bit codes for 1024 rows (byte b holds row 2b in its low nibble and row
 *       2b+1 in its high nibble; a nibble stores u = q + 8 for the signed code q in [-8, 7]),
 *       then 8 bf16 scales, one per 128-row group. Value = q * scale (symmetric).
 *   approx pool (2-bit, asymmetric, group 128): per column, ceil(d_out/512) records of 144
 *       bytes: 128 bytes of 2-bit codes for 512 rows (byte b holds rows 4b..4b+3, row r at bits
 *       2*(r%4)), then 4 little-endian uint32 words, word g = bf16 scale bits | (bf16 min bits
 *       << 16) for the record's group g. Value = min + q * scale, q in [0, 3].
 *   Rows past d_out in a column's last record are padding: 2-bit code 0 with scale = min = 0;
 *   int4 nibble 8 (q = 0) with scale 0.
 */
#ifndef SPAX_H_
#define SPAX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SPAX_ABI_VERSION 1

typedef enum {
  SPAX_OK = 0,
  SPAX_ERR_ARG = 1,        /* bad argument (NULL pointer, negative size, bad enum, bad params) */
  SPAX_ERR_SHAPE = 2,      /* unsupported shape (d_out % 128 != 0, size over a stated limit) */
  SPAX_ERR_WORKSPACE = 3,  /* workspace pointer NULL or ws_bytes too small */
  SPAX_ERR_CUDA = 4,       /* a CUDA runtime call or launch failed */
  SPAX_ERR_NONFINITE = 5,  /* device: an input activation was NaN or Inf */
  SPAX_ERR_TIMEOUT = 6,    /* device: a bounded wait ran out (a split's partial sums never
                              arrived: a library bug, or the grid could not be resident at once) */
  SPAX_ERR_INDEX = 7       /* device: counts or a column index out of range */
} spax_status;

typedef enum { SPAX_FULL_BF16 = 0, SPAX_FULL_INT4_G128 = 1 } spax_full_fmt;

typedef enum {
  SPAX_MASK_THRESHOLD = 0,
  SPAX_MASK_TOPK = 1,
  SPAX_MASK_GUIDED = 2,
  SPAX_MASK_TOPK_SCALED = 3
} spax_mask_mode;

typedef enum { SPAX_OP_TIERED_GEMV = 0, SPAX_OP_DENSE_GEMV = 1, SPAX_OP_CALIBRATE = 2 } spax_op;

/* Largest d_in a mask call accepts (the activation vector lives in one CTA's shared memory). */
#define SPAX_MASK_MAX_DIN 32768

/*
 * Tier-rule parameters for spax_build_mask.
 *   THRESHOLD (TEAL-style; TopK-Guided Abstract and §1): skip if |x| < t_skip, approximate if
 *     t_skip <= |x| < t_full, full otherwise. Requires 0 <= t_skip <= t_full.
 *   TOPK (WINA-style fixed count; TopK-Guided Abstract and §1): columns ranked by |x|, largest
 *     first, ties broken by the lower column index first; the first k_full ranks are full, the
 *     next k_approx approximate, the rest skipped. Requires k_full, k_approx >= 0 and
 *     k_full + k_approx <= d_in. t_full and t_skip are an optional guess of the |x| at rank
 *     k_full and at rank k_full + k_approx (calibrated quantiles, e.g. from
 *     spax_calibrate_thresholds at the skip fractions 1 - (k_full + k_approx)/d_in and
 *     1 - k_full/d_in): a guess within about 12% lets the kernels find the boundaries in one
 *     windowed pass instead of the full search. Any value is accepted (0, a negative, NaN or
 *     Inf means no guess), and the selected columns never depend on it. A guess that misses
 *     costs that pass (about 2 us per launch) on top of the full search, so pass none where
 *     the token-to-token scale of x varies by more than the window (or use TOPK_SCALED).
 *   TOPK_SCALED: TOPK (the same columns, lists and counts, counts[2] = counts[3] = 0) whose
 *     guesses t_full and t_skip are multiples of the token's mean key: the mean of |x| over the
 *     d_in columns (of the WINA score in spax_masked_gemv_wina). The kernels multiply them by
 *     that mean (one block reduction, fp32, fixed order) before the windowed pass, so the
 *     guess follows the token's scale. Calibrate the multiples as the quantiles divided by the
 *     mean |x| of the calibration tokens. Same requirements as TOPK. Not a rule of the pages:
 *     it only changes how fast the boundaries are found.
 *   GUIDED (TopK-Guided §2.1): the natural counts n1 = #{|x| < t_skip} and n2 = #{|x| < t_full}
 *     are clipped into the bands [ceil((s-δ)d), floor((s+δ)d)] around the skip target
 *     s = s_skip_bp/1e4 and the skip-or-approximate target s = s_below_full_bp/1e4
 *     (δ = delta_bp/1e4), giving m1 <= m2; then TOPK with k_full = d - m2,
 *     k_approx = m2 - m1. All band arithmetic is integer. Requires 0 <= s_skip_bp <=
 *     s_below_full_bp <= 10000, 0 <= delta_bp <= 10000, and the THRESHOLD requirements.
 */
typedef struct {
  int32_t mode;
  float t_skip;
  float t_full;
  int32_t k_full;
  int32_t k_approx;
  int32_t s_skip_bp;
  int32_t s_below_full_bp;
  int32_t delta_bp;
} spax_mask_params;

/*
 * A packed matrix: both pools owned by the caller, in device memory or in page-locked host
 * memory mapped into the device address space (unified addressing: the host pointer of a
 * cudaHostAlloc / cudaHostRegister allocation). With host pools the GEMV kernels read the
 * selected column segments straight over the host link, which is the offloaded-weights setting
 * of the SpAx Abstract and of the eigenradar commentary ("The route outside GPU memory"): only
 * the full and approximate tiers' bytes cross the link. Results are identical to device pools.
 */
typedef struct {
  int32_t d_out;
  int32_t d_in;
  int32_t full_fmt;  /* spax_full_fmt */
  int32_t reserved;
  const void* d_full;    /* full pool, layout above */
  const void* d_approx;  /* approx pool, layout above */
} spax_packed;

/* ABI version (SPAX_ABI_VERSION) and a static string for a status code. */
int spax_abi_version(void);
const char* spax_status_string(int status);

/*
 * Bytes of the two packed pools of a d_out × d_in matrix (host-only, no CUDA call).
 * Writes *h_full_bytes and *h_approx_bytes (either may be NULL); returns their sum, or 0 for an
 * invalid shape/format.
 */
size_t spax_pack_bytes(int d_out, int d_in, int full_fmt, size_t* h_full_bytes,
                       size_t* h_approx_bytes);

/*
 * spax_pack_weights — offline: quantise and re-lay W for the tiered GEMV.
 * Source: SpAx Abstract ("compressed weight representation"); eigenradar "two-bit approximate"
 * tier. Quantiser per column and 128-row group, in fp32 with IEEE rounding:
 *   2-bit: mn, mx = min, max of the group; min = bf16(mn); scale = bf16_rne((mx - mn) / 3);
 *          q = clamp(rint_even((w - min) / scale), 0, 3), q = 0 when scale == 0.
 *   int4:  scale = bf16_rne(max|w| / 7); q = clamp(rint_even(w / scale), -8, 7), q = 0 when
 *          scale == 0.
 * d_W: row-major [d_out][d_in] bf16 (device). d_full / d_approx: device buffers of at least
 * spax_pack_bytes() bytes each, fully written (padding included). Returns SPAX_ERR_SHAPE if
 * d_out % 128 != 0 or d_out, d_in < 1; SPAX_ERR_ARG for NULL pointers or a bad format.
 */
spax_status spax_pack_weights(const void* d_W, int d_out, int d_in, int full_fmt, void* d_full,
                              void* d_approx, void* stream);

/*
 * spax_column_norms — offline: the Euclidean norm of every column of W, for the WINA score.
 * Source: TopK-Guided §C.1 (WINA's per-element score of a column: the activation's magnitude
 * times the column's norm) and §1 (WINA's fixed-count TopK rule).
 * norm_j = fp32(sqrt(Σ_r W[r][j]^2)), the sum in fp64 in row order (each bf16 square is exact
 * in fp64), sqrt correctly rounded, then rounded to fp32: one fixed definition, so every caller
 * that follows it gets the same bits. d_W: row-major [d_out][d_in] bf16 (device); d_norms: fp32
 * [d_in] (device), fully written. SPAX_ERR_SHAPE if d_out or d_in < 1.
 */
spax_status spax_column_norms(const void* d_W, int d_out, int d_in, float* d_norms, void* stream);

/*
 * spax_calibrate_thresholds — offline: the calibrated |x| thresholds of the threshold and
 * guided rules (TopK-Guided §2.1 "calibrated threshold", §2.2 calibration pass).
 * Pools the M = n_tok * d_in values |x| of d_calib_x (row-major [n_tok][d_in] fp32) and, for
 * s = s_skip_bp/1e4 and s = s_below_full_bp/1e4, returns the order statistic of 0-based rank
 * min(floor(s*M + 1/2), M - 1) of the ascending |x| values (integer arithmetic). Writes
 * d_t_out[0] = t_skip and d_t_out[1] = t_full (device fp32). A NaN or Inf input sets
 * *d_status = SPAX_ERR_NONFINITE (thresholds are then unspecified).
 * Workspace: spax_workspace_bytes(SPAX_OP_CALIBRATE, 0, d_in) bytes of device memory, any
 * contents. Requires n_tok, d_in >= 1, n_tok * d_in < 2^31, 0 <= s_*_bp <= 10000.
 */
spax_status spax_calibrate_thresholds(const float* d_calib_x, int n_tok, int d_in, int s_skip_bp,
                                      int s_below_full_bp, float* d_t_out, int32_t* d_status,
                                      void* d_ws, size_t ws_bytes, void* stream);

/*
 * spax_build_mask — per token: the tier of every column and the compacted column lists.
 * Source: SpAx Abstract (three options chosen by activation magnitude); TopK-Guided §2.1
 * (mask construction in O(d), realised sparsity within ±δ of the target).
 * d_x: fp32 [d_in] activations. Outputs (device): d_tier uint8 [d_in] (0/1/2),
 * d_full_idx int32 [d_in] and d_approx_idx int32 [d_in] (the first counts[0] / counts[1]
 * entries are written, ascending), d_counts int32 [4] = {n_full, n_approx, n1, n2} with n1, n2
 * the natural threshold counts (0 for TOPK). A NaN/Inf in x sets *d_status =
 * SPAX_ERR_NONFINITE, every tier to 0 and the counts to 0. h_params is a host pointer, read
 * during the call. d_in <= SPAX_MASK_MAX_DIN. One CTA; no workspace.
 */
spax_status spax_build_mask(const float* d_x, int d_in, const spax_mask_params* h_params,
                            uint8_t* d_tier, int32_t* d_full_idx, int32_t* d_approx_idx,
                            int32_t* d_counts, int32_t* d_status, void* stream);

/*
 * spax_tiered_gemv — per token: y = Σ_{j in full} x_j W[:,j] + Σ_{j in approx} x_j deq2(W)[:,j].
 * Source: SpAx Abstract (read original weights for the largest |x|, approximate weights for
 * smaller, skip the rest); eigenradar commentary (bytes moved per token; reconstruction of
 * two-bit approximations costs GPU time).
 * h_W: host pointer to the packed-matrix descriptor (device pools). d_x fp32 [d_in];
 * d_full_idx / d_approx_idx / d_counts as written by spax_build_mask (the kernel reads
 * counts on the device; no host sync). d_y fp32 [d_out] (device), fully written.
 * Accumulation is fp32, split over CTAs, then reduced in a fixed order (bit-reproducible for a
 * given GPU model and shape). Workspace: spax_workspace_bytes(SPAX_OP_TIERED_GEMV, d_out, d_in)
 * bytes, ZEROED BEFORE FIRST USE: it holds the split-K partial sums as flagged words that every
 * completed call leaves at zero (zero it again after a device error). Counts outside [0, d_in]
 * or an index outside [0, d_in) set *d_status = SPAX_ERR_INDEX; such a column contributes zero.
 * Calls that share a workspace must not run concurrently.
 * Residency: the CTAs that split a row tile wait for one another's partial sums (a wait bounded
 * at 1 s, then SPAX_ERR_TIMEOUT and an unspecified y). The launch is one wave of at most one CTA
 * per SM and needs its whole grid resident at once, which holds when the call has the GPU's SMs
 * to itself: no kernel of another stream or process holding SMs while it runs, and no context
 * limited to a subset of the SMs (MPS thread limits, green contexts).
 */
spax_status spax_tiered_gemv(const spax_packed* h_W, const float* d_x, const int32_t* d_full_idx,
                             const int32_t* d_approx_idx, const int32_t* d_counts, float* d_y,
                             int32_t* d_status, void* d_ws, size_t ws_bytes, void* stream);

/*
 * spax_masked_gemv — spax_build_mask and spax_tiered_gemv for one token in a single launch.
 * Source: SpAx Abstract (three tiers by activation magnitude); TopK-Guided §1 and §2.1 (the
 * threshold, TopK and guided rules); eigenradar commentary (bytes moved per token).
 * Every CTA of the GEMV computes the token's tiers and ordered lists itself (the same rule, same
 * results as spax_build_mask) and reads its split's columns from its own copy, so the lists never
 * make a round trip through global memory and no second launch is needed.
 * h_W, d_x, d_y, d_status, d_ws, ws_bytes: as spax_tiered_gemv (same workspace size and rules).
 * h_params: host pointer, as spax_build_mask. d_tier, d_full_idx, d_approx_idx, d_counts: the
 * mask's outputs, written exactly as spax_build_mask writes them; each may be NULL (not written).
 * A NaN/Inf in x sets *d_status = SPAX_ERR_NONFINITE, the tiers and counts to 0 and y to 0.
 * Requires d_in <= SPAX_MASK_MAX_DIN and the shared memory of the shape's plan to fit one CTA
 * (else SPAX_ERR_SHAPE; every d_in up to 28672 fits).
 */
spax_status spax_masked_gemv(const spax_packed* h_W, const float* d_x,
                             const spax_mask_params* h_params, float* d_y, uint8_t* d_tier,
                             int32_t* d_full_idx, int32_t* d_approx_idx, int32_t* d_counts,
                             int32_t* d_status, void* d_ws, size_t ws_bytes, void* stream);

/*
 * spax_masked_gemv_swiglu — spax_masked_gemv whose activation is formed in the kernel from the
 * gated-MLP pair before it: x_j = silu(g_j) * u_j with silu(g) = g / (1 + e^-g), for the down
 * projection fed straight from the tiered gate/up output. Source: the same passages as
 * spax_masked_gemv; the chained gate/up -> down step is the decoder layer around them.
 * d_gu: fp32 [2 * d_in] (device) = [g_0 .. g_{d_in-1}, u_0 .. u_{d_in-1}], i.e. the y of a gate/up
 * matrix packed as gate rows then up rows. x_j is computed in fp32 (IEEE divide and multiply, the
 * library's expf) by one function wherever the kernel needs it, so the tier rule and the product
 * see the same value. d_x_out: fp32 [d_in] (device) receives that x; may be NULL. Every other
 * argument, output and rule as spax_masked_gemv; a non-finite x_j (from a non-finite g or u, or
 * an overflowing product) is SPAX_ERR_NONFINITE.
 */
/*
 * spax_masked_gemv_wina — spax_masked_gemv whose rule ranks columns by the WINA score
 * s_j = |x_j| * norm_j instead of |x_j|. Source: TopK-Guided §1 (WINA's TopK rule) and §C.1
 * (its per-element score: activation magnitude times the column norm).
 * d_norms: fp32 [d_in] (device), as spax_column_norms writes them. The score is one correctly
 * rounded fp32 product; every rule (threshold, TopK, guided) and tie order of spax_build_mask
 * then applies to s in place of |x| (thresholds, and a TopK guess of the boundary keys, are on
 * s). The product still uses x. A
 * non-finite score is SPAX_ERR_NONFINITE. Every other argument, output and rule as
 * spax_masked_gemv.
 */
spax_status spax_masked_gemv_wina(const spax_packed* h_W, const float* d_x,
                                  const float* d_norms, const spax_mask_params* h_params,
                                  float* d_y, uint8_t* d_tier, int32_t* d_full_idx,
                                  int32_t* d_approx_idx, int32_t* d_counts, int32_t* d_status,
                                  void* d_ws, size_t ws_bytes, void* stream);

spax_status spax_masked_gemv_swiglu(const spax_packed* h_W, const float* d_gu,
                                    const spax_mask_params* h_params, float* d_y, float* d_x_out,
                                    uint8_t* d_tier, int32_t* d_full_idx, int32_t* d_approx_idx,
                                    int32_t* d_counts, int32_t* d_status, void* d_ws,
                                    size_t ws_bytes, void* stream);

/*
 * spax_test_tiered_gemv_timeout — failure-detection test hook, not a computation. It launches
 * the list-driven GEMV of spax_tiered_gemv with the last column split of every row tile left
 * out, so the CTAs that wait for that split's partial sums give up after wait_limit_ns and set
 * *d_status = SPAX_ERR_TIMEOUT, leaving the context usable. Afterwards y is unspecified and the
 * scratch holds flagged words: zero the workspace (or call spax_fixed_scratch_reset) before the
 * next GEMV. d_ws NULL selects the fixed scratch array of spax_tiered_gemv_fixed_scratch.
 * Requires a shape whose plan has at least 2 splits (SPAX_ERR_SHAPE otherwise) and
 * 1e6 <= wait_limit_ns <= 2e9. Other arguments as spax_tiered_gemv.
 */
spax_status spax_test_tiered_gemv_timeout(const spax_packed* h_W, const float* d_x,
                                          const int32_t* d_full_idx, const int32_t* d_approx_idx,
                                          const int32_t* d_counts, float* d_y, int32_t* d_status,
                                          void* d_ws, size_t ws_bytes, uint64_t wait_limit_ns,
                                          void* stream);

/*
 * spax_dense_gemv — the same-GPU dense baseline: y = W x over every column, read from the
 * bf16 full pool (W^T [d_in][d_out]) with the same kernel family as spax_tiered_gemv.
 * Source: eigenradar commentary (comparisons use dense decoding in the same weight format).
 * Workspace: spax_workspace_bytes(SPAX_OP_DENSE_GEMV, d_out, d_in) bytes, zeroed before first
 * use (same rule as spax_tiered_gemv). d_out % 128 == 0.
 */
spax_status spax_dense_gemv(const void* d_Wt, const float* d_x, float* d_y, int d_out, int d_in,
                            int32_t* d_status, void* d_ws, size_t ws_bytes, void* stream);

/*
 * spax_tiered_gemv_fixed_scratch — the same computation as spax_tiered_gemv (same arguments
 * minus the workspace, same results, same kernel), for callers that cannot allocate device
 * memory where they call it: its split-K scratch is a fixed array compiled into the library
 * (spax_fixed_scratch_bytes() = 4 MiB per device), so the call allocates nothing. The pages
 * have no counterpart of this entry point; it is an interface convenience.
 * - The first call in each device's context (with that device current) looks up the array's
 *   device address and caches it; make that first call before any stream capture on that
 *   device. The cache is keyed on the context's process-unique id, so after a cudaDeviceReset
 *   the next call looks the address up again (the new context's array starts at zero).
 * - Shapes whose split plan needs more partial sums than the array holds are rejected with
 *   SPAX_ERR_WORKSPACE before anything is launched (none on a 148-SM GPU: a plan with splits
 *   needs at most S * d_out * 8 <= 148 * 2048 * 8 bytes, and one without needs none).
 * - The array starts at zero when the library loads and every completed call leaves it at zero.
 *   A call that ends in a device error (SPAX_ERR_TIMEOUT, or a sticky CUDA error) may leave
 *   flagged partial sums in it, which a later call would take for its own: after any such error,
 *   call spax_fixed_scratch_reset before the next fixed-scratch call.
 * - There is ONE array per device for the whole process: calls on the same device that can
 *   overlap (other streams, other threads, concurrent graph branches) race on it and give
 *   wrong results. Serialise them.
 * - Like spax_tiered_gemv, the launch needs its whole grid (one CTA per SM) resident at once:
 *   see the residency note there.
 */
spax_status spax_tiered_gemv_fixed_scratch(const spax_packed* h_W, const float* d_x,
                                           const int32_t* d_full_idx, const int32_t* d_approx_idx,
                                           const int32_t* d_counts, float* d_y, int32_t* d_status,
                                           void* stream);

/*
 * spax_fixed_scratch_reset — zero the current device's fixed scratch array (one
 * cudaMemsetAsync on `stream`; allocates nothing). Call it after a fixed-scratch call reported
 * SPAX_ERR_TIMEOUT or any device error, ordered after that call and before the next one.
 */
spax_status spax_fixed_scratch_reset(void* stream);

/* Size in bytes of the per-device scratch array spax_tiered_gemv_fixed_scratch uses. */
size_t spax_fixed_scratch_bytes(void);

/*
 * Device workspace bytes an op needs for a shape on the CURRENT device (the split count
 * depends on its SM count), enough for either full-tier format. Returns 0 for an invalid op or
 * shape.
 */
size_t spax_workspace_bytes(int op, int d_out, int d_in);

/*
 * Host-only: the split-K factor S and row tile R the tiered/dense GEMV uses for a shape on the
 * current device (for reporting and tests). Returns SPAX_ERR_SHAPE/ARG on a bad shape.
 */
spax_status spax_gemv_plan(int op, int d_out, int d_in, int full_fmt, int32_t* h_splits,
                           int32_t* h_row_tile);

/*
 * spax_output_change — d_acc[0] += Σ_i (y_i - y_ref_i)^2 and d_acc[1] += Σ_i y_ref_i^2 over the n
 * entries of two device vectors, in fp64, by one CTA in a fixed order (the same bits on every
 * run). d_acc: two doubles on the device, accumulated into (the caller zeroes them).
 * Source: TopK-Guided §2.2 (block sensitivity as the output change at a probe sparsity).
 */
spax_status spax_output_change(const float* d_y, const float* d_y_ref, int n, double* d_acc,
                               void* stream);

/*
 * spax_probe_sensitivity — offline: how far one matrix's output moves when its input is
 * sparsified to the probe sparsity s̄ = s_probe_bp / 1e4 (TopK-Guided §2.2: each block's
 * sensitivity is measured as its output change at a probe sparsity; the budgets then follow from
 * spax_block_budgets). For each calibration token x_t (row t of d_X, row-major [n_tok][d_in]):
 * y_ref = the masked GEMV with every column in full (the matrix's own full-tier format) and y =
 * the masked GEMV with the TopK rule k_full = d_in - floor(s̄ d_in + 1/2), k_approx = 0 (the
 * smallest |x| skipped, the rest in full); then spax_output_change(y, y_ref) into d_acc. A
 * block's sensitivity is sqrt(Σ_m acc0_m / Σ_m acc1_m) over its matrices m. At s̄ = 0 both
 * products take the same columns in the same order, so acc0 gains exactly 0.
 * d_y2: device scratch of 2 * d_out floats (the second half 16-byte aligned); d_ws / ws_bytes:
 * the tiered GEMV's workspace (zeroed before first use). Launches 3 * n_tok kernels on stream.
 */
spax_status spax_probe_sensitivity(const spax_packed* h_W, const float* d_X, int n_tok,
                                   int s_probe_bp, float* d_y2, double* d_acc, int32_t* d_status,
                                   void* d_ws, size_t ws_bytes, void* stream);

/*
 * Host-only, no CUDA call: the plan of op for a GPU with sm_count SMs (the split count S, the row
 * tile R and the workspace bytes), by the same rule the calls use on the current device. For
 * sizing workspaces for another GPU model, and for checking a shape against
 * spax_fixed_scratch_bytes(): spax_tiered_gemv_fixed_scratch rejects exactly the shapes whose
 * SPAX_OP_TIERED_GEMV plan needs more workspace than that (SPAX_ERR_WORKSPACE).
 */
spax_status spax_gemv_plan_sms(int op, int d_out, int d_in, int full_fmt, int sm_count,
                               int32_t* h_splits, int32_t* h_row_tile, size_t* h_ws_bytes);

/*
 * spax_block_budgets — host-only: sensitivity-aware per-block sparsity (TopK-Guided §2.2:
 * above-average-sensitivity blocks get less sparsity, λ sets the redistribution, results are
 * clamped to [lo, hi], the global budget is kept). With σ̄ the mean of h_sens:
 *   s_b = clamp(s * (1 - λ (σ_b/σ̄ - 1)) + c, lo, hi), c chosen so that mean_b s_b = s.
 * h_sens: n_blocks positive sensitivities; writes h_s_out[n_blocks]. Requires lo <= s <= hi,
 * 0 <= lo <= hi <= 1, λ >= 0, n_blocks >= 1.
 */
spax_status spax_block_budgets(const double* h_sens, int n_blocks, double s, double lambda,
                               double lo, double hi, double* h_s_out);

/*
 * Block output reconstruction error for the per-matrix sparsities h_p[0, n) of one block
 * (measured by the caller, e.g. on calibration tokens); ctx is passed through unchanged.
 */
typedef double (*spax_block_error_fn)(const double* h_p, int n, void* ctx);

/*
 * spax_greedy_allocation — host-only: per-matrix sparsities inside one block, given the block's
 * budget (TopK-Guided, Appendix D "Block-wise Greedy Sparsity Allocation", and Table 4).
 * Matrix m has parameter count h_params[m] = f_m and step alpha_m = alpha * fbar / f_m (fbar
 * the mean count), so one increment of any matrix moves the compute-weighted block sparsity
 * P = sum_m f_m p_m / sum_m f_m by alpha / n. From p = 0, each step tries the next increment of
 * every matrix whose p_m + alpha_m stays <= p_max, evaluates err on each candidate allocation,
 * and keeps the candidate with the least error (ties: the lower matrix index). It stops as soon
 * as P >= p_target - 1e-12. Writes h_p_out[n], *h_steps and, when h_order is not NULL, the
 * matrix chosen at each step (h_order holds max_steps entries).
 * Requires n >= 1, every f_m > 0, alpha > 0, 0 <= p_target <= p_max <= 1 and err != NULL.
 * Returns SPAX_ERR_ARG if the budget cannot be reached within max_steps steps or before every
 * matrix is at p_max (the allocation reached so far is still written).
 */
spax_status spax_greedy_allocation(const double* h_params, int n, double alpha, double p_target,
                                   double p_max, spax_block_error_fn err, void* ctx,
                                   int max_steps, double* h_p_out, int32_t* h_order,
                                   int32_t* h_steps);

/*
 * Host-only byte account of one tiered GEMV (eigenradar "bytes moved per generated token"):
 * weight bytes the kernel must read for n_full full and n_approx approximate columns of a
 * d_out-row matrix: n_full * (2*d_out for bf16 | 0.5*d_out + 2*d_out/128 for int4) +
 * n_approx * (d_out/4 + 4*d_out/128). Returns 0 on a bad shape.
 */
uint64_t spax_weight_bytes(int d_out, int full_fmt, int64_t n_full, int64_t n_approx);

#ifdef __cplusplus
}
#endif
#endif /* SPAX_H_ */
