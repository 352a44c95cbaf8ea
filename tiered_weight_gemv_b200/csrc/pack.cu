// pack.cu — offline packing of a row-major bf16 matrix into the tiered GEMV's column pools.
//
// Sources: SpAx (arXiv 2610.02598), Abstract — a compressed weight representation read for
// small-magnitude activations; eigenradar commentary on SpAx — a two-bit approximate tier.
// Quantiser per column and 128-row group, fp32 with IEEE rounding (explicit _rn intrinsics, no
// contraction), codes taken against the STORED bf16 scale/min:
//   2-bit asymmetric: min = bf16(mn); scale = bf16_rne((mx - mn) / 3);
//                     q = clamp(rint_even((w - min) / scale), 0, 3)   (q = 0 if scale == 0)
//   int4 symmetric:   scale = bf16_rne(max|w| / 7); q = clamp(rint_even(w / scale), -8, 7)
// Layout (see spax.h): bf16 pool = W^T; int4 pool = per column 528-byte records of 1024 rows;
// 2-bit pool = per column 144-byte records of 512 rows. Padding rows are written too.
//
// One thread handles one (column, 128-row group); a warp spans 32 consecutive columns, so each
// row read is a coalesced 64-byte segment of the row-major input.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace spax {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }
__device__ __forceinline__ uint32_t f32_to_bf16_bits(float f) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

template <int FMT>
__global__ void __launch_bounds__(256) pack_kernel(const uint16_t* __restrict__ W, int d_out,
                                                   int d_in, uint8_t* full, uint8_t* approx,
                                                   int groups_total) {
  pdl_wait();
  pdl_launch_dependents();
  const int j = blockIdx.x * 32 + (threadIdx.x & 31);
  const int g = blockIdx.y * 8 + (threadIdx.x >> 5);
  if (j >= d_in || g >= groups_total) return;
  const int G = d_out / 128;
  const long long stride2 = (long long)((d_out + 511) / 512) * 144;
  const long long stride4 = (long long)((d_out + 1023) / 1024) * 528;
  const int nrec2_groups = ((d_out + 511) / 512) * 4;
  const int nrec4_groups = ((d_out + 1023) / 1024) * 8;

  uint32_t w[64];  // the group's 128 bf16 values, two per word (row 2i low, 2i+1 high)
  if (g < G) {
    const uint16_t* src = W + (long long)g * 128 * d_in + j;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      const uint32_t lo = __ldg(src + (long long)(2 * i) * d_in);
      const uint32_t hi = __ldg(src + (long long)(2 * i + 1) * d_in);
      w[i] = lo | (hi << 16);
    }
  }

  // ---- 2-bit approx pool ----
  if (g < nrec2_groups) {
    uint8_t* rec = approx + (long long)j * stride2 + (long long)(g / 4) * 144;
    uint32_t codes[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // 128 rows x 2 bits
    uint32_t smw = 0u;
    if (g < G) {
      float mn = bf16_bits_to_f32(w[0] & 0xFFFFu), mx = mn;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const float a = bf16_bits_to_f32(w[i] & 0xFFFFu), b = bf16_bits_to_f32(w[i] >> 16);
        mn = fminf(mn, fminf(a, b));
        mx = fmaxf(mx, fmaxf(a, b));
      }
      mn = __fadd_rn(mn, 0.0f);  // a zero extreme is +0, whatever fminf/fmaxf returned
      mx = __fadd_rn(mx, 0.0f);
      const uint32_t sb = f32_to_bf16_bits(__fdiv_rn(__fsub_rn(mx, mn), 3.0f));
      const uint32_t mb = f32_to_bf16_bits(mn);
      const float s = bf16_bits_to_f32(sb), m = bf16_bits_to_f32(mb);
#pragma unroll
      for (int i = 0; i < 64; ++i) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float v = bf16_bits_to_f32(h ? (w[i] >> 16) : (w[i] & 0xFFFFu));
          int q = 0;
          if (s != 0.0f) q = min(3, max(0, __float2int_rn(__fdiv_rn(__fsub_rn(v, m), s))));
          const int r = 2 * i + h;  // row within the group: word r/16, bits 2*(r%16)
          codes[r >> 4] |= static_cast<uint32_t>(q) << (2 * (r & 15));
        }
      }
      smw = sb | (mb << 16);
    }
    uint4* cdst = reinterpret_cast<uint4*>(rec + (g % 4) * 32);
    cdst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
    cdst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
    reinterpret_cast<uint32_t*>(rec + 128)[g % 4] = smw;
  }

  // ---- full pool ----
  if constexpr (FMT == SPAX_FULL_BF16) {
    if (g < G) {
      uint4* dst = reinterpret_cast<uint4*>(full + ((long long)j * d_out + (long long)g * 128) * 2);
#pragma unroll
      for (int i = 0; i < 16; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
  } else {
    if (g < nrec4_groups) {
      uint8_t* rec = full + (long long)j * stride4 + (long long)(g / 8) * 528;
      uint32_t nib[16];  // 128 rows x 4 bits, row r at bits 4*(r%8) of word r/8
#pragma unroll
      for (int i = 0; i < 16; ++i) nib[i] = 0x88888888u;
      uint32_t sb = 0u;
      if (g < G) {
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 64; ++i)
          amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_f32(w[i] & 0xFFFFu)), fabsf(bf16_bits_to_f32(w[i] >> 16))));
        sb = f32_to_bf16_bits(__fdiv_rn(amax, 7.0f));
        const float s = bf16_bits_to_f32(sb);
#pragma unroll
        for (int i = 0; i < 16; ++i) nib[i] = 0u;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float v = bf16_bits_to_f32(h ? (w[i] >> 16) : (w[i] & 0xFFFFu));
            int q = 0;
            if (s != 0.0f) q = min(7, max(-8, __float2int_rn(__fdiv_rn(v, s))));
            const int r = 2 * i + h;
            nib[r >> 3] |= static_cast<uint32_t>(q + 8) << (4 * (r & 7));
          }
        }
      }
      uint4* cdst = reinterpret_cast<uint4*>(rec + (g % 8) * 64);
#pragma unroll
      for (int i = 0; i < 4; ++i) cdst[i] = make_uint4(nib[4 * i], nib[4 * i + 1], nib[4 * i + 2], nib[4 * i + 3]);
      reinterpret_cast<uint16_t*>(rec + 512)[g % 8] = static_cast<uint16_t>(sb);
    }
  }
}

// Column norms for the WINA score (TopK-Guided §C.1): one thread per column sums the squares of
// its d_out bf16 values in fp64, in row order (a fixed order: every square is exact in fp64, the
// sum rounds the same way wherever this definition is followed), then a correctly rounded sqrt
// and one rounding to fp32. The loads of eight rows are issued together; a warp reads 32
// neighbouring columns of a row (64 contiguous bytes).
__global__ void __launch_bounds__(256) column_norm_kernel(const uint16_t* __restrict__ W,
                                                         int d_out, int d_in,
                                                         float* __restrict__ norms) {
  pdl_wait();
  pdl_launch_dependents();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d_in) return;
  const uint16_t* col = W + j;
  double acc = 0.0;
  int r = 0;
  for (; r + 8 <= d_out; r += 8) {
    uint16_t v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = __ldg(col + (size_t)(r + k) * d_in);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const double w = (double)__uint_as_float((uint32_t)v[k] << 16);
      acc = __dadd_rn(acc, __dmul_rn(w, w));
    }
  }
  for (; r < d_out; ++r) {
    const double w = (double)__uint_as_float((uint32_t)__ldg(col + (size_t)r * d_in) << 16);
    acc = __dadd_rn(acc, __dmul_rn(w, w));
  }
  norms[j] = __double2float_rn(__dsqrt_rn(acc));
}

cudaError_t launch_column_norms(const void* W, int d_out, int d_in, float* norms,
                                cudaStream_t stream) {
  return launch_pdl(column_norm_kernel, dim3((d_in + 255) / 256), dim3(256), 0, stream,
                    static_cast<const uint16_t*>(W), d_out, d_in, norms);
}

cudaError_t launch_pack(const void* W, int d_out, int d_in, int full_fmt, void* full, void* approx,
                        cudaStream_t stream) {
  const int nrec2_groups = ((d_out + 511) / 512) * 4;
  const int nrec4_groups = ((d_out + 1023) / 1024) * 8;
  const int groups_total = full_fmt == SPAX_FULL_BF16 ? nrec2_groups : max(nrec2_groups, nrec4_groups);
  const dim3 grid((d_in + 31) / 32, (groups_total + 7) / 8);
  const auto* w16 = static_cast<const uint16_t*>(W);
  auto* f8 = static_cast<uint8_t*>(full);
  auto* a8 = static_cast<uint8_t*>(approx);
  if (full_fmt == SPAX_FULL_BF16)
    return launch_pdl(pack_kernel<SPAX_FULL_BF16>, grid, dim3(256), 0, stream, w16, d_out, d_in,
                      f8, a8, groups_total);
  return launch_pdl(pack_kernel<SPAX_FULL_INT4_G128>, grid, dim3(256), 0, stream, w16, d_out,
                    d_in, f8, a8, groups_total);
}

}  // namespace spax
