// mask.cu — per-token tier of every column and the compacted column lists (one CTA).
//
// Sources: SpAx (arXiv 2610.02598), Abstract; TopK-Guided (arXiv 2610.01763), Abstract, §1 and
// §2.1. The rule itself (rank order, boundaries, selection and compaction) lives in select.cuh;
// this kernel runs it and writes the tier codes, both ascending lists and the counts.
#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace spax {

size_t mask_smem_bytes(int d) { return select_keys_bytes(d) + select_list_bytes(d); }

__global__ void __launch_bounds__(kSelThreads, 1)
    mask_kernel(const float* __restrict__ x, int d, spax_mask_params prm, uint8_t* __restrict__ tier,
                int32_t* __restrict__ full_idx, int32_t* __restrict__ approx_idx,
                int32_t* __restrict__ counts, int32_t* status) {
  extern __shared__ __align__(16) uint32_t keys[];
  __shared__ __align__(16) SelectSmem S;
  select_zero(S);
  pdl_wait();
  pdl_launch_dependents();
  select_fetch(x, d, keys);  // its barrier also orders the zeroing above
  uint32_t n1, n2;
  Boundary B[2];
  // TOPK_SCALED: its guesses become keys first (the token's mean key times the multiples), so
  // the kernel holds one copy of the rule
  const spax_mask_params rule =
      prm.mode == SPAX_MASK_TOPK_SCALED ? select_scaled_topk(prm, d, keys, S) : prm;
  if (select_rule(rule, d, keys, S, &n1, &n2, B)) {
    for (int j = threadIdx.x; j < d; j += kSelThreads) tier[j] = 0;
    if (threadIdx.x == 0) {
      counts[0] = counts[1] = counts[2] = counts[3] = 0;
      record_status(status, SPAX_ERR_NONFINITE);
    }
    return;
  }
  uint16_t* list = reinterpret_cast<uint16_t*>(keys + 4 * ((d + 3) / 4));
  uint32_t nf, na, a0;
  select_compact(keys, d, B, S, tier, list, &nf, &na, &a0);
  select_write_lists(list, d, nf, na, a0, full_idx, approx_idx);
  if (threadIdx.x == 0) {
    counts[0] = (int32_t)nf;
    counts[1] = (int32_t)na;
    const bool topk = prm.mode == SPAX_MASK_TOPK || prm.mode == SPAX_MASK_TOPK_SCALED;
    counts[2] = topk ? 0 : (int32_t)n1;
    counts[3] = topk ? 0 : (int32_t)n2;
  }
}

cudaError_t launch_mask(const float* x, int d_in, const spax_mask_params& p, uint8_t* tier,
                        int32_t* full_idx, int32_t* approx_idx, int32_t* counts, int32_t* status,
                        cudaStream_t stream) {
  const int smem = (int)mask_smem_bytes(d_in);
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(mask_kernel), smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(mask_kernel, dim3(1), dim3(kSelThreads), (size_t)smem, stream, x, d_in, p,
                    tier, full_idx, approx_idx, counts, status);
}

}  // namespace spax
