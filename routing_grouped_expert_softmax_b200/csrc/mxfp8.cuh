// MXFP8 element and scale arithmetic shared by the quantisers (quant.cu) and the grouped
// GEMM epilogues that quantise their own outputs (grouped_gemm.cu): OCP Microscaling
// Formats (MX) v1.0, E4M3 elements with one E8M0 scale per 32 elements, X = 2^(floor(log2
// amax) - 8), elements rounded to nearest even and saturated to +-448.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

// E8M0 exponent s (scale 2^s) of a block from its largest magnitude.
__device__ __forceinline__ int mx_scale_exp(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int e = (int)((bits >> 23) & 0xFF);
  if (e == 0) return -127;                 // zero or fp32-subnormal amax
  return max(e - 127 - 8, -127);           // floor(log2 amax) - 8 (at most 119 for finite amax)
}

// 2^-s as a float, for s in [-127, 119]
__device__ __forceinline__ float exp2_neg(int s) { return __uint_as_float((uint32_t)(127 - s) << 23); }

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  return (uint16_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

// Scale layouts.  Plain: K-major operands [rows][K/32], token-axis operands [rows/32][cols].
// Tiled (what the block-scaled GEMMs read, one 512-byte bulk copy per operand and pipeline
// stage): tiles of 128 rows (or columns) of the MMA's M or N dimension by 4 consecutive
// K-blocks; tile (mn/128, kb/4) sits at ((mn/128) * nkg + kb/4) * 512, nkg = the K extent in
// 128-element groups, and inside it the scale of (mn, kb) is byte 16*(mn%32) + 4*((mn%128)/32)
// + kb%4: the arrangement tcgen05.cp's 32x128b.warpx4 copy reads (32 rows of 16 bytes, row
// mn%32 holding the four K-blocks of mn%32, mn%32 + 32, + 64, + 96).
__device__ __forceinline__ int64_t sf_tiled_off(int64_t mn, int64_t kb, int64_t nkg) {
  return ((mn >> 7) * nkg + (kb >> 2)) * 512 + 16 * (mn & 31) + 4 * ((mn & 127) >> 5) + (kb & 3);
}

// Quantise 32 values (one block along K, held by this thread) and store their 32 codes at
// `codes` (16-byte aligned) and their scale byte at `scale`.
__device__ __forceinline__ void mx_block32_store(const float (&v)[32], uint8_t *codes, uint8_t *scale) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int sc = mx_scale_exp(amax);
  const float inv = exp2_neg(sc);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = (uint32_t)e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv) |
           ((uint32_t)e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv) << 16);
  uint4 *d4 = reinterpret_cast<uint4 *>(codes);
  d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
  d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
  *scale = (uint8_t)(sc + 127);
}

// A 32 x 32 slab held one row per lane (lane l: row l, values v): quantise each column as one
// block of 32 rows (the block maximum of column i is the warp's maximum of |v[i]|; for
// non-negative floats the bit patterns order as unsigned integers, so one redux.sync per
// column).  Lane l stores its row's 32 codes at `codes` (16-byte aligned) and the scale byte
// of column l at `scale`.  Every lane of the warp must call it.
__device__ __forceinline__ void mx_slab32_cols_store(const float (&v)[32], uint8_t *codes, uint8_t *scale) {
  const int lane = threadIdx.x & 31;
  uint32_t w[8];
  int mine = 0;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float a0 = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v[i]))));
    const float a1 = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v[i + 1]))));
    const int s0 = mx_scale_exp(a0), s1 = mx_scale_exp(a1);
    if (lane == i) mine = s0;
    if (lane == i + 1) mine = s1;
    const uint32_t pair = e4m3x2(v[i] * exp2_neg(s0), v[i + 1] * exp2_neg(s1));
    if (i & 2) w[i >> 2] |= pair << 16; else w[i >> 2] = pair;
  }
  uint4 *d4 = reinterpret_cast<uint4 *>(codes);
  d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
  d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
  *scale = (uint8_t)(mine + 127);
}

}  // namespace moe
