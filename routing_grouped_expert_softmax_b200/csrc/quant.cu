// MXFP8 quantisers: E4M3 elements with one E8M0 power-of-two scale per 32 elements along a
// GEMM's reduction axis.
//
// Method: unite.ai "Ai2 κυκλοφορεί το Olmo-Core 3 ...", section "Παραλληλισμός, Ακρίβεια
// και Τεχνικές Μνήμης" (MXFP8 on selected operations, chiefly the feed-forward compute and
// the data moved between experts).  Formats: OCP Microscaling Formats (MX) v1.0 — for a
// block with largest magnitude amax, X = 2^(floor(log2 amax) - 8) (8 = exponent of E4M3's
// largest normal, 448 = 1.75 * 2^8), clamped to E8M0's [2^-127, 2^127]; amax = 0 gives
// 2^-127; each element is v / X rounded to nearest-even E4M3 and saturated to +-448.
//
// Two block directions:
//   rows  — blocks of 32 consecutive columns of a row (K runs along the row);
//           codes [R][K], scales [R][K/32];
//   cols  — blocks of 32 consecutive rows of a column (K runs down the rows, the
//           token axis of the weight-gradient GEMMs); codes [R][C], scales [R/32][C].
// Activation operands are written into expert buffers padded to 128 rows: padded row
// 128*pre[e] + i holds source row offsets[e] + i for i < count_e and zeros after, where
// pre[e] = sum_{e' < e} ceil(count_e' / 128).
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

// Padded-row bookkeeping: exclusive prefix of 128-row blocks per expert, by one warp.
__device__ void mx_block_prefix(const int32_t *offsets, int E, int *pre) {
  const int lane = threadIdx.x & 31;
  int cnt[8], sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int e = lane * 8 + i;
    cnt[i] = (e < E) ? (offsets[e + 1] - offsets[e] + 127) / 128 : 0;
    sum += cnt[i];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int run = incl - sum;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int e = lane * 8 + i;
    if (e < E) pre[e] = run;
    run += cnt[i];
  }
  if (lane == 31) pre[E] = incl;
}

// Source row of padded row pr, or -1 for a pad row / a row past the end.
__device__ __forceinline__ int64_t mx_src_row(int64_t pr, const int32_t *offsets, const int *pre, int E) {
  const int g = (int)(pr >> 7);
  if (g >= pre[E]) return -1;
  int lo = 0, hi = E;  // pre[lo] <= g < pre[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (pre[mid] <= g) lo = mid; else hi = mid;
  }
  const int64_t local = pr - (int64_t)pre[lo] * 128;
  const int cnt = offsets[lo + 1] - offsets[lo];
  return local < cnt ? (int64_t)offsets[lo] + local : -1;
}

// ---- rows: one warp per (row, 1024-column chunk); lane l owns the 32-column block l.
// offsets == nullptr: identity row map over R rows.
__global__ void __launch_bounds__(256) mx_quant_rows_kernel(const bf16 *__restrict__ src, int64_t R, int K,
                                                            const int32_t *__restrict__ offsets, int E,
                                                            uint8_t *__restrict__ codes,
                                                            uint8_t *__restrict__ scales) {
  __shared__ int pre[MAX_E + 1];
  if (offsets) {
    if (threadIdx.x < 32) mx_block_prefix(offsets, E, pre);
    __syncthreads();
  }
  const int lane = threadIdx.x & 31;
  const int64_t pr = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int64_t rows_out = offsets ? (int64_t)pre[E] * 128 : R;
  if (pr >= rows_out) return;
  const int64_t sr = offsets ? mx_src_row(pr, offsets, pre, E) : pr;
  for (int c0 = blockIdx.y * 1024; c0 < K; c0 += gridDim.y * 1024) {
    const int blk = c0 / 32 + lane;
    if (c0 + lane * 32 >= K) break;
    uint4 raw[4];
    if (sr >= 0) {
      const uint4 *s4 = reinterpret_cast<const uint4 *>(src + sr * K + c0 + lane * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) raw[i] = __ldg(s4 + i);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) raw[i] = make_uint4(0, 0, 0, 0);
    }
    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) Vec<bf16>::load(raw[i], &v[8 * i]);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int s = mx_scale_exp(amax);
    const float inv = exp2_neg(s);
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      w[i] = (uint32_t)e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv) |
             ((uint32_t)e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv) << 16);
    uint4 *d4 = reinterpret_cast<uint4 *>(codes + pr * K + c0 + lane * 32);
    d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
    d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
    scales[pr * (K / 32) + blk] = (uint8_t)(s + 127);
  }
}

// Four adjacent columns of a 32-row block: reads 8 bytes of every row (one warp reads 256
// contiguous bytes per row) once for the block maxima and again (from cache) to quantise,
// and stores 4 code bytes per row and the 4 scale bytes.
__device__ __forceinline__ uint2 mx_row8(const bf16 *src, int64_t ld_src, int i, int nvalid) {
  return i < nvalid ? __ldg(reinterpret_cast<const uint2 *>(src + i * ld_src)) : make_uint2(0u, 0u);
}
__device__ __forceinline__ void mx_cols4(const bf16 *src, int64_t ld_src, int nvalid, uint8_t *codes,
                                         int64_t ld_codes, uint8_t *scales) {
  float amax[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint2 r = mx_row8(src, ld_src, i, nvalid);
    amax[0] = fmaxf(amax[0], fabsf(__uint_as_float(r.x << 16)));
    amax[1] = fmaxf(amax[1], fabsf(__uint_as_float(r.x & 0xFFFF0000u)));
    amax[2] = fmaxf(amax[2], fabsf(__uint_as_float(r.y << 16)));
    amax[3] = fmaxf(amax[3], fabsf(__uint_as_float(r.y & 0xFFFF0000u)));
  }
  int sc[4];
  float inv[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    sc[j] = mx_scale_exp(amax[j]);
    inv[j] = exp2_neg(sc[j]);
  }
#pragma unroll 8
  for (int i = 0; i < 32; ++i) {
    const uint2 r = mx_row8(src, ld_src, i, nvalid);
    const uint32_t w =
        (uint32_t)e4m3x2(__uint_as_float(r.x << 16) * inv[0], __uint_as_float(r.x & 0xFFFF0000u) * inv[1]) |
        ((uint32_t)e4m3x2(__uint_as_float(r.y << 16) * inv[2], __uint_as_float(r.y & 0xFFFF0000u) * inv[3]) << 16);
    *reinterpret_cast<uint32_t *>(codes + i * ld_codes) = w;
  }
  *reinterpret_cast<uint32_t *>(scales) = (uint32_t)(sc[0] + 127) | ((uint32_t)(sc[1] + 127) << 8) |
                                          ((uint32_t)(sc[2] + 127) << 16) | ((uint32_t)(sc[3] + 127) << 24);
}

// ---- cols: one thread per (4 adjacent columns, 32-row block).  C % 4 == 0.
__global__ void __launch_bounds__(256) mx_quant_cols_kernel(const bf16 *__restrict__ src, int64_t R, int C,
                                                            const int32_t *__restrict__ offsets, int E,
                                                            uint8_t *__restrict__ codes,
                                                            uint8_t *__restrict__ scales) {
  __shared__ int pre[MAX_E + 1];
  if (offsets) {
    if (threadIdx.x < 32) mx_block_prefix(offsets, E, pre);
    __syncthreads();
  }
  const int c = 4 * (blockIdx.x * 256 + threadIdx.x);
  const int64_t rb = blockIdx.y;                       // 32-row block
  const int64_t rows_out = offsets ? (int64_t)pre[E] * 128 : R;
  if (rb * 32 >= rows_out || c >= C) return;
  // all 32 rows of a block belong to one expert (experts are padded to 128 rows)
  int64_t sr0 = offsets ? mx_src_row(rb * 32, offsets, pre, E) : rb * 32;
  int nvalid = offsets ? 32 : (int)(R - rb * 32 < 32 ? R - rb * 32 : 32);
  if (offsets) {
    if (sr0 < 0) nvalid = 0;
    else {
      // rows of this block still inside the expert
      const int g = (int)((rb * 32) >> 7);
      int lo = 0, hi = E;
      while (hi - lo > 1) { int mid = (lo + hi) >> 1; if (pre[mid] <= g) lo = mid; else hi = mid; }
      const int64_t local = rb * 32 - (int64_t)pre[lo] * 128;
      const int64_t left = offsets[lo + 1] - offsets[lo] - local;
      nvalid = (int)(left < 32 ? left : 32);
    }
  }
  if (sr0 < 0) sr0 = 0;   // nothing is read from it then
  mx_cols4(src + sr0 * C + c, C, nvalid, codes + rb * 32 * C + c, C, scales + rb * C + c);
}

// ---- weights of the gate/up GEMM, blocked down the rows, with gate and up columns
// interleaved in 64-column chunks: output column 128*j + i is gate column 64*j + i for
// i < 64 and up column 64*j + (i - 64) otherwise.  src: W_gate, W_up [R][f].  One thread per
// 4 adjacent output columns (never split across a 64-column chunk) and 32-row block.
__global__ void __launch_bounds__(256) mx_quant_cols_gu_kernel(const bf16 *__restrict__ wg,
                                                               const bf16 *__restrict__ wu, int64_t R, int f,
                                                               uint8_t *__restrict__ codes,
                                                               uint8_t *__restrict__ scales) {
  const int oc = 4 * (blockIdx.x * 256 + threadIdx.x);   // output column in [0, 2f)
  const int64_t rb = blockIdx.y;
  if (oc >= 2 * f || rb * 32 >= R) return;
  const int j = oc >> 7, i = oc & 127;
  const bf16 *src = i < 64 ? wg : wu;
  const int c = 64 * j + (i & 63);
  const int nvalid = (int)(R - rb * 32 < 32 ? R - rb * 32 : 32);
  mx_cols4(src + rb * 32 * f + c, f, nvalid, codes + rb * 32 * (2 * f) + oc, 2 * f, scales + rb * (2 * f) + oc);
}

// ---- weights of the gate/up data-gradient GEMM, blocked along the rows of [W_gate | W_up]
// (K = 2f): row r of the output is [W_gate[r] | W_up[r]].
__global__ void __launch_bounds__(256) mx_quant_rows_gu_kernel(const bf16 *__restrict__ wg,
                                                               const bf16 *__restrict__ wu, int64_t R, int f,
                                                               uint8_t *__restrict__ codes,
                                                               uint8_t *__restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= R) return;
  const int K = 2 * f;
  for (int c0 = 0; c0 < K; c0 += 1024) {
    const int col = c0 + lane * 32;
    if (col >= K) break;
    const bf16 *s = col < f ? wg + r * f + col : wu + r * f + (col - f);
    const uint4 *s4 = reinterpret_cast<const uint4 *>(s);
    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) Vec<bf16>::load(__ldg(s4 + i), &v[8 * i]);
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
    uint4 *d4 = reinterpret_cast<uint4 *>(codes + r * K + col);
    d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
    d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
    scales[r * (K / 32) + col / 32] = (uint8_t)(sc + 127);
  }
}

// ---- FP8 dispatch: x_perm[slot(t,j)] = x[t] (a bit copy) and, in the same pass, the row in
// MXFP8 (blocks of 32 along d) at padded row 128*pre[e] + (slot - offsets[e]) of the expert
// buffers, e the expert holding the slot.  One warp per token; lane l quantises the 32-column
// blocks l, l+32, ... once and writes them to all k destinations.  Padded rows past an
// expert's count are not written (the gate/up GEMM computes and drops them).
__global__ void __launch_bounds__(256) mx_permute_kernel(const bf16 *__restrict__ x, const int32_t *__restrict__ sop,
                                                         const int32_t *__restrict__ offsets, int E, int64_t T,
                                                         int k, int d, bf16 *__restrict__ x_perm,
                                                         uint8_t *__restrict__ codes, uint8_t *__restrict__ scales) {
  __shared__ int pre[MAX_E + 1];
  if (threadIdx.x < 32) mx_block_prefix(offsets, E, pre);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  int64_t my_slot = 0, my_prow = 0;
  if (lane < k) {
    my_slot = sop[t * k + lane];
    int lo = 0, hi = E;   // the expert whose range holds the slot: offsets[lo] <= slot < offsets[lo + 1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (offsets[mid] <= my_slot) lo = mid; else hi = mid;
    }
    my_prow = (int64_t)pre[lo] * 128 + (my_slot - offsets[lo]);
  }
  int64_t slot[MAX_K], prow[MAX_K];
#pragma unroll
  for (int j = 0; j < MAX_K; ++j) {
    slot[j] = __shfl_sync(0xffffffffu, my_slot, j);
    prow[j] = __shfl_sync(0xffffffffu, my_prow, j);
  }
  for (int c0 = 0; c0 < d; c0 += 1024) {
    const int col = c0 + lane * 32;
    if (col >= d) break;
    const uint4 *s4 = reinterpret_cast<const uint4 *>(x + t * d + col);
    uint4 raw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) raw[i] = __ldg(s4 + i);
    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) Vec<bf16>::load(raw[i], &v[8 * i]);
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
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) {
      if (j < k) {
        uint4 *xp = reinterpret_cast<uint4 *>(x_perm + slot[j] * d + col);
#pragma unroll
        for (int i = 0; i < 4; ++i) xp[i] = raw[i];
        uint4 *d4 = reinterpret_cast<uint4 *>(codes + prow[j] * d + col);
        d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
        scales[prow[j] * (d / 32) + col / 32] = (uint8_t)(sc + 127);
      }
    }
  }
}

cudaError_t launch_mx_permute(const void *x, const int32_t *sop, const int32_t *offsets, int E, int64_t T, int k,
                              int d, void *x_perm, uint8_t *codes, uint8_t *scales, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  mx_permute_kernel<<<(unsigned)((T + 7) / 8), 256, 0, st>>>(static_cast<const bf16 *>(x), sop, offsets, E, T, k, d,
                                                             static_cast<bf16 *>(x_perm), codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_mx_quant_rows(const void *src, int64_t R, int K, const int32_t *offsets, int E, int64_t rows_bound,
                                 uint8_t *codes, uint8_t *scales, cudaStream_t st) {
  if (rows_bound <= 0) return cudaSuccess;
  dim3 grid((unsigned)((rows_bound + 7) / 8), (unsigned)((K + 1023) / 1024));
  mx_quant_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const bf16 *>(src), R, K, offsets, E, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_mx_quant_cols(const void *src, int64_t R, int C, const int32_t *offsets, int E, int64_t rows_bound,
                                 uint8_t *codes, uint8_t *scales, cudaStream_t st) {
  if (rows_bound <= 0) return cudaSuccess;
  dim3 grid((unsigned)((C / 4 + 255) / 256), (unsigned)((rows_bound + 31) / 32));
  mx_quant_cols_kernel<<<grid, 256, 0, st>>>(static_cast<const bf16 *>(src), R, C, offsets, E, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_mx_quant_cols_gu(const void *wg, const void *wu, int64_t R, int f, uint8_t *codes,
                                    uint8_t *scales, cudaStream_t st) {
  dim3 grid((unsigned)((2 * f / 4 + 255) / 256), (unsigned)((R + 31) / 32));
  mx_quant_cols_gu_kernel<<<grid, 256, 0, st>>>(static_cast<const bf16 *>(wg), static_cast<const bf16 *>(wu), R, f,
                                                codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_mx_quant_rows_gu(const void *wg, const void *wu, int64_t R, int f, uint8_t *codes,
                                    uint8_t *scales, cudaStream_t st) {
  mx_quant_rows_gu_kernel<<<(unsigned)((R + 7) / 8), 256, 0, st>>>(static_cast<const bf16 *>(wg),
                                                                    static_cast<const bf16 *>(wu), R, f, codes,
                                                                    scales);
  return cudaGetLastError();
}

}  // namespace moe
