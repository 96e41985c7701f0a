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
#include <atomic>

#include "common.cuh"
#include "mxfp8.cuh"

namespace moe {

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
                                                            uint8_t *__restrict__ scales, bool tiled) {
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
    scales[tiled ? sf_tiled_off(pr, blk, K / 128) : pr * (K / 32) + blk] = (uint8_t)(s + 127);
  }
}

// Four adjacent columns of a 32-row block: reads 8 bytes of every row (one warp reads 256
// contiguous bytes per row) once for the block maxima and again (from cache) to quantise,
// and stores 4 code bytes per row and the 4 scale bytes.
__device__ __forceinline__ uint2 mx_row8(const bf16 *src, int64_t ld_src, int i, int nvalid) {
  return i < nvalid ? __ldg(reinterpret_cast<const uint2 *>(src + i * ld_src)) : make_uint2(0u, 0u);
}
__device__ __forceinline__ uint32_t mx_cols4(const bf16 *src, int64_t ld_src, int nvalid, uint8_t *codes,
                                             int64_t ld_codes) {
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
  // the four columns' scale bytes, column j in byte j
  return (uint32_t)(sc[0] + 127) | ((uint32_t)(sc[1] + 127) << 8) | ((uint32_t)(sc[2] + 127) << 16) |
         ((uint32_t)(sc[3] + 127) << 24);
}

// Scale bytes of four adjacent columns c..c+3 (K-block kb): plain, one 4-byte store at
// row kb of [.][C]; tiled, one byte each.
__device__ __forceinline__ void mx_put_scales4(uint8_t *scales, uint32_t sc4, int64_t kb, int c, int C, bool tiled,
                                               int64_t nkg) {
  if (!tiled) {
    *reinterpret_cast<uint32_t *>(scales + kb * C + c) = sc4;
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) scales[sf_tiled_off(c + j, kb, nkg)] = (uint8_t)(sc4 >> (8 * j));
  }
}

// ---- cols: one thread per (4 adjacent columns, 32-row block).  C % 4 == 0.
__global__ void __launch_bounds__(256) mx_quant_cols_kernel(const bf16 *__restrict__ src, int64_t R, int C,
                                                            const int32_t *__restrict__ offsets, int E,
                                                            uint8_t *__restrict__ codes,
                                                            uint8_t *__restrict__ scales, bool tiled, int64_t nkg) {
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
  const uint32_t sc4 = mx_cols4(src + sr0 * C + c, C, nvalid, codes + rb * 32 * C + c, C);
  mx_put_scales4(scales, sc4, rb, c, C, tiled, nkg);
}

// ---- weights of the gate/up GEMM, blocked down the rows, with gate and up columns
// interleaved in 64-column chunks: output column 128*j + i is gate column 64*j + i for
// i < 64 and up column 64*j + (i - 64) otherwise.  src: W_gate, W_up [R][f].  One thread per
// 4 adjacent output columns (never split across a 64-column chunk) and 32-row block.
__global__ void __launch_bounds__(256) mx_quant_cols_gu_kernel(const bf16 *__restrict__ wg,
                                                               const bf16 *__restrict__ wu, int64_t R, int f,
                                                               uint8_t *__restrict__ codes,
                                                               uint8_t *__restrict__ scales, bool tiled) {
  const int oc = 4 * (blockIdx.x * 256 + threadIdx.x);   // output column in [0, 2f)
  const int64_t rb = blockIdx.y;
  if (oc >= 2 * f || rb * 32 >= R) return;
  const int j = oc >> 7, i = oc & 127;
  const bf16 *src = i < 64 ? wg : wu;
  const int c = 64 * j + (i & 63);
  const int nvalid = (int)(R - rb * 32 < 32 ? R - rb * 32 : 32);
  const uint32_t sc4 = mx_cols4(src + rb * 32 * f + c, f, nvalid, codes + rb * 32 * (2 * f) + oc, 2 * f);
  mx_put_scales4(scales, sc4, rb, oc, 2 * f, tiled, (R + 127) / 128);
}

// ---- weights of the gate/up data-gradient GEMM, blocked along the rows of [W_gate | W_up]
// (K = 2f): row r of the output is [W_gate[r] | W_up[r]].
__global__ void __launch_bounds__(256) mx_quant_rows_gu_kernel(const bf16 *__restrict__ wg,
                                                               const bf16 *__restrict__ wu, int64_t R, int f,
                                                               uint8_t *__restrict__ codes,
                                                               uint8_t *__restrict__ scales, bool tiled) {
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
    scales[tiled ? sf_tiled_off(r, col / 32, K / 128) : r * (K / 32) + col / 32] = (uint8_t)(sc + 127);
  }
}

// ---- weights in both orientations from one read.  A block takes 128 rows and NC "tile
// columns": for the gate/up pair (gu) 128 columns of W_gate and the same 128 of W_up (NC = 256,
// in the interleaved output order below), else NC = 256 (or 128 when C % 256 != 0) columns of
// one tensor [R][C].  From the tile it writes
//   codes_c: blocks of 32 down the rows (the forward GEMMs' K), [R][C'] with C' = 2f for the
//            pair (gate and up interleaved in 64-column chunks: output column 128 J + i is gate
//            column 64 J + i for i < 64, up column 64 J + i - 64 otherwise) or C;
//   codes_r: blocks of 32 along the row (the data-gradient GEMMs' K), [R][C'] with row r of the
//            pair [W_gate[r] | W_up[r]];
// and the scales of both in the tile layout.  128 rows hold four 32-row blocks and NC columns
// whole 128-column groups, so the block owns whole 512-byte scale tiles: it assembles them in
// shared memory and writes them with 16-byte stores.  Same arithmetic as the single-orientation
// kernels (block maxima of the bf16 values, scale rule, E4M3 rounding).
constexpr int WQ_ROWS = 128, WQ_THREADS = 512, WQ_NC_MAX = 256, WQ_PAD = 8;
constexpr size_t WQ_TILE_BYTES = (size_t)WQ_ROWS * (WQ_NC_MAX + WQ_PAD) * 2;
// the tile, the inverse scales and the two staged scale tiles of each orientation (two blocks
// fit on an SM)
constexpr size_t WQ_SMEM = WQ_TILE_BYTES + 4 * WQ_NC_MAX * 4 + WQ_ROWS * (WQ_NC_MAX / 32) * 4 + 2 * 2 * 512;

struct WqMap {
  bool gu;
  int C, NC, c0;
  // source tensor (0 or 1) and column of tile column j
  __device__ __forceinline__ int tensor(int j) const { return gu ? (j >> 6) & 1 : 0; }
  __device__ __forceinline__ int src_col(int j) const { return gu ? c0 + 64 * (j >> 7) + (j & 63) : c0 + j; }
  // output column of tile column j: column-blocked (interleaved for the pair) and row-blocked
  __device__ __forceinline__ int ccol(int j) const { return gu ? 2 * c0 + j : c0 + j; }
  __device__ __forceinline__ int rcol(int j) const { return tensor(j) * C + src_col(j); }
};

// One block per tile (tile column block blockIdx.x, row block blockIdx.y).
template <bool GU, int NC>
__global__ void __launch_bounds__(WQ_THREADS) mx_quant_weights_kernel(
    const bf16 *__restrict__ w0, const bf16 *__restrict__ w1, int64_t R, int C,
    uint8_t *__restrict__ codes_c, uint8_t *__restrict__ scales_c, uint8_t *__restrict__ codes_r,
    uint8_t *__restrict__ scales_r) {
  extern __shared__ __align__(16) uint8_t wq_smem[];
  constexpr bool gu = GU;
  constexpr int pitch = NC + WQ_PAD;                                    // bf16 elements per row
  bf16 *tile = reinterpret_cast<bf16 *>(wq_smem);                       // [128][pitch]
  float *inv_c = reinterpret_cast<float *>(wq_smem + WQ_TILE_BYTES);    // [4][NC]
  float *inv_r = inv_c + 4 * NC;                                        // [128][NC/32]
  uint8_t *st_c = reinterpret_cast<uint8_t *>(inv_r + WQ_ROWS * (NC / 32));   // [NC/128][512]
  uint8_t *st_r = st_c + (NC / 128) * 512;                              // [NC/128][512]
  const WqMap m{gu, C, NC, (int)blockIdx.x * (gu ? 128 : NC)};
  const int t = threadIdx.x;
  const int64_t r0 = (int64_t)blockIdx.y * WQ_ROWS;
  const int CO = gu ? 2 * C : C;
  // (1) the tile, 16-byte pieces (8 tile columns of one chunk each): every load of the thread
  // in flight at once, then the shared-memory stores.  Piece q of thread t is row t/vpr +
  // q*(WQ_THREADS/vpr), columns 8*(t%vpr)..+7, so the four pieces of a 32-column block of a
  // row sit in four adjacent lanes: the row scales come from the registers, by two shuffles.
  constexpr int vpr = NC / 8, NLD = WQ_ROWS * vpr / WQ_THREADS;
  constexpr int nb = NC / 32;
  uint4 ld[NLD];
#pragma unroll
  for (int q = 0; q < NLD; ++q) {
    const int idx = t + q * WQ_THREADS, row = idx / vpr, j = (idx - row * vpr) * 8;
    const bf16 *w = m.tensor(j) ? w1 : w0;
    ld[q] = __ldg(reinterpret_cast<const uint4 *>(w + (r0 + row) * C + m.src_col(j)));
  }
#pragma unroll
  for (int q = 0; q < NLD; ++q) {
    const int idx = t + q * WQ_THREADS, row = idx / vpr, j = (idx - row * vpr) * 8;
    *reinterpret_cast<uint4 *>(tile + row * pitch + j) = ld[q];
    float v[8];
    Vec<bf16>::load(ld[q], v);
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    if ((t & 3) == 0) {
      const int b = j / 32;
      const int sc = mx_scale_exp(amax);
      inv_r[row * nb + b] = exp2_neg(sc);
      const int kb = m.rcol(j) / 32;                                    // K-block along the row
      const int ti = gu ? m.tensor(j) : (j >> 7);                       // which staged tile
      st_r[ti * 512 + 16 * (row & 31) + 4 * (row >> 5) + (kb & 3)] = (uint8_t)(sc + 127);
    }
  }
  __syncthreads();
  // (2) column scales: 4 row groups x NC columns, two adjacent columns per task (32 paired
  // loads)
  for (int u = t; u < 2 * NC; u += WQ_THREADS) {
    const int grp = u / (NC / 2), j = 2 * (u - grp * (NC / 2));
    float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
    for (int r = 0; r < 32; ++r) {
      const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(tile + (grp * 32 + r) * pitch + j));
      a0 = fmaxf(a0, fabsf(v.x));
      a1 = fmaxf(a1, fabsf(v.y));
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int sc = mx_scale_exp(h ? a1 : a0);
      inv_c[grp * NC + j + h] = exp2_neg(sc);
      const int mn = m.ccol(j + h) & 127;                               // the tile's base is a multiple of 128
      st_c[((j + h) >> 7) * 512 + 16 * (mn & 31) + 4 * (mn >> 5) + grp] = (uint8_t)(sc + 127);
    }
  }
  __syncthreads();
  // (3) the staged scale tiles, whole, with 16-byte stores
  for (int u = t; u < 2 * (NC / 128) * 32; u += WQ_THREADS) {
    const int which = u / ((NC / 128) * 32), rest = u - which * (NC / 128) * 32, ti = rest >> 5, q = rest & 31;
    if (which == 0) {
      const int64_t mnb = m.ccol(ti * 128) / 128, kg = r0 / 128;
      reinterpret_cast<uint4 *>(scales_c + (mnb * (R / 128) + kg) * 512)[q] =
          reinterpret_cast<const uint4 *>(st_c + ti * 512)[q];
    } else {
      const int64_t mnb = r0 / 128, kg = m.rcol(gu ? ti * 64 : ti * 128) / 128;
      reinterpret_cast<uint4 *>(scales_r + (mnb * (CO / 128) + kg) * 512)[q] =
          reinterpret_cast<const uint4 *>(st_r + ti * 512)[q];
    }
  }
  // (4) codes in both orientations: thread t takes 16 tile columns of RPT consecutive rows of
  // one 32-row group, so that the 16 column scales it needs are read once for all of them
  constexpr int TPR = NC / 16, RPT = WQ_ROWS * TPR / WQ_THREADS;
  static_assert(32 % RPT == 0, "a thread's rows lie in one row group");
  const int j0 = (t % TPR) * 16, row0 = (t / TPR) * RPT, grp = row0 >> 5;
  float ic[16];
#pragma unroll
  for (int i = 0; i < 16; i += 4) {
    const float4 f = *reinterpret_cast<const float4 *>(inv_c + grp * NC + j0 + i);
    ic[i] = f.x; ic[i + 1] = f.y; ic[i + 2] = f.z; ic[i + 3] = f.w;
  }
#pragma unroll
  for (int rr = 0; rr < RPT; ++rr) {
    const int row = row0 + rr;
    float v[16];
    Vec<bf16>::load(*reinterpret_cast<const uint4 *>(tile + row * pitch + j0), v);
    Vec<bf16>::load(*reinterpret_cast<const uint4 *>(tile + row * pitch + j0 + 8), v + 8);
    const float ir = inv_r[row * nb + j0 / 32];
    uint32_t wc[4], wr[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      wc[q] = (uint32_t)e4m3x2(v[4 * q] * ic[4 * q], v[4 * q + 1] * ic[4 * q + 1]) |
              ((uint32_t)e4m3x2(v[4 * q + 2] * ic[4 * q + 2], v[4 * q + 3] * ic[4 * q + 3]) << 16);
      wr[q] = (uint32_t)e4m3x2(v[4 * q] * ir, v[4 * q + 1] * ir) |
              ((uint32_t)e4m3x2(v[4 * q + 2] * ir, v[4 * q + 3] * ir) << 16);
    }
    *reinterpret_cast<uint4 *>(codes_c + (r0 + row) * CO + m.ccol(j0)) = make_uint4(wc[0], wc[1], wc[2], wc[3]);
    *reinterpret_cast<uint4 *>(codes_r + (r0 + row) * CO + m.rcol(j0)) = make_uint4(wr[0], wr[1], wr[2], wr[3]);
  }
}

template <bool GU, int NC>
static cudaError_t launch_wq(const void *w0, const void *w1, int64_t R, int C, uint8_t *codes_c, uint8_t *scales_c,
                             uint8_t *codes_r, uint8_t *scales_r, cudaStream_t st) {
  // the dynamic shared-memory opt-in is a per-device property of the kernel
  static std::atomic<uint64_t> attr_set{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!(attr_set.load(std::memory_order_acquire) >> dev & 1ull)) {
    cudaError_t e = cudaFuncSetAttribute(mx_quant_weights_kernel<GU, NC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)WQ_SMEM);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(1ull << dev, std::memory_order_acq_rel);
  }
  dim3 grid((unsigned)(GU ? C / 128 : C / NC), (unsigned)(R / WQ_ROWS));
  if (grid.x == 0 || grid.y == 0) return cudaSuccess;
  mx_quant_weights_kernel<GU, NC><<<grid, WQ_THREADS, WQ_SMEM, st>>>(
      static_cast<const bf16 *>(w0), static_cast<const bf16 *>(w1), R, C, codes_c, scales_c, codes_r, scales_r);
  return cudaGetLastError();
}

cudaError_t launch_mx_quant_weights(const void *w0, const void *w1, int64_t R, int C, bool gu, uint8_t *codes_c,
                                    uint8_t *scales_c, uint8_t *codes_r, uint8_t *scales_r, cudaStream_t st) {
  if (gu) return launch_wq<true, 256>(w0, w1, R, C, codes_c, scales_c, codes_r, scales_r, st);
  if (C % 256 == 0) return launch_wq<false, 256>(w0, w1, R, C, codes_c, scales_c, codes_r, scales_r, st);
  return launch_wq<false, 128>(w0, w1, R, C, codes_c, scales_c, codes_r, scales_r, st);
}

// ---- FP8 dispatch: x_perm[slot(t,j)] = x[t] (a bit copy) and, in the same pass, the row in
// MXFP8 (blocks of 32 along d) at padded row 128*pre[e] + (slot - offsets[e]) of the expert
// buffers, e the expert holding the slot.  One warp per token; lane l quantises the 32-column
// blocks l, l+32, ... once and writes them to all k destinations.  Padded rows past an
// expert's count are not written (the gate/up GEMM computes and drops them).
__global__ void __launch_bounds__(256) mx_permute_kernel(const bf16 *__restrict__ x, const int32_t *__restrict__ sop,
                                                         const int32_t *__restrict__ offsets, int E, int64_t T,
                                                         int k, int d, bf16 *__restrict__ x_perm,
                                                         uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
                                                         bool tiled) {
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
        scales[tiled ? sf_tiled_off(prow[j], col / 32, d / 128) : prow[j] * (d / 32) + col / 32] =
            (uint8_t)(sc + 127);
      }
    }
  }
}

// ---- Slot-major FP8 dispatch, forward and backward.  One block per 32 padded rows of one
// expert; warp w takes rows 4w..4w+3; the columns go in chunks of 256, 8 per lane.  For the
// routed pair in slot s (token t, gate g) the row is
//   forward (BWD = false):  x_perm[s] = x[t]             (src = x; a bit copy)
//   backward (BWD = true):  dy_perm[s] = bf16(g dY[t])    (src = dY), dgate = <dY[t], y_perm[s]>
// and in the same pass the row in MXFP8 along d (codes_r, blocks of 32 columns; may be null)
// and down the token axis (codes_c, blocks of 32 rows of the expert-padded layout), scales in
// the GEMMs' tile layout (tiled) or plain ([rows][d/32] and [rows/32][d]).  out_perm may be
// null (the bf16 rows are not written).  Pad rows are zeros.
constexpr int CB_CHUNK = 256;
template <bool BWD>
__global__ void __launch_bounds__(256, 2) mx_slot_dispatch_kernel(
    const bf16 *__restrict__ src, const bf16 *__restrict__ y_perm, const int32_t *__restrict__ pos,
    const int32_t *__restrict__ offsets, const float *__restrict__ gate, int E, int k, int d, int64_t nkt,
    bf16 *__restrict__ out_perm, float *__restrict__ dgate, uint8_t *__restrict__ codes_r,
    uint8_t *__restrict__ scales_r, uint8_t *__restrict__ codes_c, uint8_t *__restrict__ scales_c, bool tiled) {
  __shared__ int pre[MAX_E + 1];
  __shared__ float colmax[8][CB_CHUNK];
  __shared__ float inv_col[CB_CHUNK];
  if (threadIdx.x < 32) mx_block_prefix(offsets, E, pre);
  __syncthreads();
  const int64_t blk = blockIdx.x;                    // 32-row block of the padded layout
  if (blk * 32 >= (int64_t)pre[E] * 128) return;     // (uniform over the block)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this block's expert: pre[e] <= blk / 4 < pre[e + 1]
  const int g = (int)(blk >> 2);
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pre[mid] <= g) lo = mid; else hi = mid;
  }
  const int cnt = offsets[lo + 1] - offsets[lo];
  int prow[4], tok[4], pair[4];   // (row and slot counts stay below 2^31)
  float gt[4], dot[4];
  bool valid[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    prow[i] = (int)blk * 32 + warp * 4 + i;
    const int local = prow[i] - pre[lo] * 128;
    valid[i] = local < cnt;
    const int slot = offsets[lo] + (valid[i] ? local : 0);
    pair[i] = valid[i] ? pos[slot] : 0;
    tok[i] = pair[i] / k;
    gt[i] = (BWD && valid[i]) ? gate[pair[i]] : 0.f;
    dot[i] = 0.f;
  }
  // The rows' 16-byte pieces of chunk c0 + CB_CHUNK are loaded while chunk c0 is quantised
  // (its three block barriers would otherwise leave no load in flight).
  int slot_of[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) slot_of[i] = offsets[lo] + (prow[i] - pre[lo] * 128);
  uint4 nx[4], ny[4] = {};
  auto fetch = [&](int c0n) {
    const int cn = c0n + lane * 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool on = valid[i] && cn < d;
      nx[i] = on ? __ldg(reinterpret_cast<const uint4 *>(src + (int64_t)tok[i] * d + cn)) : make_uint4(0, 0, 0, 0);
      if constexpr (BWD)
        ny[i] = on ? __ldg(reinterpret_cast<const uint4 *>(y_perm + (int64_t)slot_of[i] * d + cn))
                   : make_uint4(0, 0, 0, 0);
    }
  };
  // the forward's blocks take one chunk each (grid.y = chunks); the backward's blocks walk the
  // whole row, whose dot product with y_perm gives dgate
  const int c_lo = BWD ? 0 : (int)blockIdx.y * CB_CHUNK, c_hi = BWD ? d : min(d, c_lo + CB_CHUNK);
  fetch(c_lo);
  for (int c0 = c_lo; c0 < c_hi; c0 += CB_CHUNK) {
    const int c = c0 + lane * 8;
    const bool cin = c < d;       // d % 128 == 0: a 32-column block is wholly in or out
    uint4 cx[4], cy[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) { cx[i] = nx[i]; cy[i] = ny[i]; }
    if (BWD && c0 + CB_CHUNK < c_hi) fetch(c0 + CB_CHUNK);
    float v[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t slot = slot_of[i];
      if (valid[i] && cin) {
        const uint4 raw = cx[i];
        if constexpr (BWD) {
          float fd[8], fy[8];
          Vec<bf16>::load(raw, fd);
          Vec<bf16>::load(cy[i], fy);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            dot[i] = fmaf(fd[j], fy[j], dot[i]);
            v[i][j] = gt[i] * fd[j];
          }
          const uint4 o = Vec<bf16>::store(v[i]);                // the bf16 dy_perm row
          if (out_perm) *reinterpret_cast<uint4 *>(out_perm + slot * d + c) = o;
          Vec<bf16>::load(o, v[i]);
        } else {
          if (out_perm) *reinterpret_cast<uint4 *>(out_perm + slot * d + c) = raw;   // a bit copy
          Vec<bf16>::load(raw, v[i]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[i][j] = 0.f;
      }
    }
    // along d: a block of 32 columns is 4 lanes x 8
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float amax = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[i][j]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      const int sc = mx_scale_exp(amax);
      const float inv = exp2_neg(sc);
      uint2 w;
      w.x = (uint32_t)e4m3x2(v[i][0] * inv, v[i][1] * inv) | ((uint32_t)e4m3x2(v[i][2] * inv, v[i][3] * inv) << 16);
      w.y = (uint32_t)e4m3x2(v[i][4] * inv, v[i][5] * inv) | ((uint32_t)e4m3x2(v[i][6] * inv, v[i][7] * inv) << 16);
      if (cin && codes_r) {
        *reinterpret_cast<uint2 *>(codes_r + (int64_t)prow[i] * d + c) = w;
        if ((lane & 3) == 0)
          scales_r[tiled ? sf_tiled_off(prow[i], c / 32, d / 128) : (int64_t)prow[i] * (d / 32) + c / 32] =
              (uint8_t)(sc + 127);
      }
    }
    // down the token axis: the block's 32 rows of each column
#pragma unroll
    for (int j = 0; j < 8; ++j)
      colmax[warp][lane * 8 + j] =
          fmaxf(fmaxf(fabsf(v[0][j]), fabsf(v[1][j])), fmaxf(fabsf(v[2][j]), fabsf(v[3][j])));
    __syncthreads();
    {
      float amax = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) amax = fmaxf(amax, colmax[w][threadIdx.x]);
      const int sc = mx_scale_exp(amax);
      inv_col[threadIdx.x] = exp2_neg(sc);
      if (c0 + (int)threadIdx.x < d)
        scales_c[tiled ? sf_tiled_off(c0 + threadIdx.x, blk, nkt) : blk * d + c0 + threadIdx.x] = (uint8_t)(sc + 127);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float *iv = &inv_col[lane * 8];
      uint2 w;
      w.x = (uint32_t)e4m3x2(v[i][0] * iv[0], v[i][1] * iv[1]) | ((uint32_t)e4m3x2(v[i][2] * iv[2], v[i][3] * iv[3]) << 16);
      w.y = (uint32_t)e4m3x2(v[i][4] * iv[4], v[i][5] * iv[5]) | ((uint32_t)e4m3x2(v[i][6] * iv[6], v[i][7] * iv[7]) << 16);
      if (cin) *reinterpret_cast<uint2 *>(codes_c + (int64_t)prow[i] * d + c) = w;
    }
    __syncthreads();   // colmax and inv_col are rewritten by the next chunk
  }
  if constexpr (BWD) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float s = dot[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0 && valid[i]) dgate[pair[i]] = s;
    }
  }
}

cudaError_t launch_mx_combine_bwd(const void *dy, const void *y_perm, const int32_t *pos, const int32_t *offsets,
                                  const float *gate, int E, int k, int d, int64_t rows_bound, void *dy_perm,
                                  float *dgate, uint8_t *codes_r, uint8_t *scales_r, uint8_t *codes_c,
                                  uint8_t *scales_c, cudaStream_t st, bool tiled) {
  if (rows_bound <= 0) return cudaSuccess;
  mx_slot_dispatch_kernel<true><<<(unsigned)((rows_bound + 31) / 32), 256, 0, st>>>(
      static_cast<const bf16 *>(dy), static_cast<const bf16 *>(y_perm), pos, offsets, gate, E, k, d,
      (rows_bound + 127) / 128, static_cast<bf16 *>(dy_perm), dgate, codes_r, scales_r, codes_c, scales_c, tiled);
  return cudaGetLastError();
}

cudaError_t launch_mx_dispatch(const void *x, const int32_t *pos, const int32_t *offsets, int E, int k, int d,
                               int64_t rows_bound, void *x_perm, uint8_t *codes_r, uint8_t *scales_r,
                               uint8_t *codes_c, uint8_t *scales_c, cudaStream_t st, bool tiled) {
  if (rows_bound <= 0) return cudaSuccess;
  const dim3 grid((unsigned)((rows_bound + 31) / 32), (unsigned)((d + CB_CHUNK - 1) / CB_CHUNK));
  mx_slot_dispatch_kernel<false><<<grid, 256, 0, st>>>(
      static_cast<const bf16 *>(x), nullptr, pos, offsets, nullptr, E, k, d, (rows_bound + 127) / 128,
      static_cast<bf16 *>(x_perm), nullptr, codes_r, scales_r, codes_c, scales_c, tiled);
  return cudaGetLastError();
}

cudaError_t launch_mx_permute(const void *x, const int32_t *sop, const int32_t *offsets, int E, int64_t T, int k,
                              int d, void *x_perm, uint8_t *codes, uint8_t *scales, cudaStream_t st, bool tiled) {
  if (T == 0) return cudaSuccess;
  mx_permute_kernel<<<(unsigned)((T + 7) / 8), 256, 0, st>>>(static_cast<const bf16 *>(x), sop, offsets, E, T, k, d,
                                                             static_cast<bf16 *>(x_perm), codes, scales, tiled);
  return cudaGetLastError();
}

cudaError_t launch_mx_quant_rows(const void *src, int64_t R, int K, const int32_t *offsets, int E, int64_t rows_bound,
                                 uint8_t *codes, uint8_t *scales, cudaStream_t st, bool tiled) {
  if (rows_bound <= 0) return cudaSuccess;
  dim3 grid((unsigned)((rows_bound + 7) / 8), (unsigned)((K + 1023) / 1024));
  mx_quant_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const bf16 *>(src), R, K, offsets, E, codes, scales, tiled);
  return cudaGetLastError();
}

cudaError_t launch_mx_quant_cols(const void *src, int64_t R, int C, const int32_t *offsets, int E, int64_t rows_bound,
                                 uint8_t *codes, uint8_t *scales, cudaStream_t st, bool tiled) {
  if (rows_bound <= 0) return cudaSuccess;
  dim3 grid((unsigned)((C / 4 + 255) / 256), (unsigned)((rows_bound + 31) / 32));
  mx_quant_cols_kernel<<<grid, 256, 0, st>>>(static_cast<const bf16 *>(src), R, C, offsets, E, codes, scales, tiled,
                                             (rows_bound + 127) / 128);
  return cudaGetLastError();
}

cudaError_t launch_mx_quant_cols_gu(const void *wg, const void *wu, int64_t R, int f, uint8_t *codes,
                                    uint8_t *scales, cudaStream_t st, bool tiled) {
  dim3 grid((unsigned)((2 * f / 4 + 255) / 256), (unsigned)((R + 31) / 32));
  mx_quant_cols_gu_kernel<<<grid, 256, 0, st>>>(static_cast<const bf16 *>(wg), static_cast<const bf16 *>(wu), R, f,
                                                codes, scales, tiled);
  return cudaGetLastError();
}

cudaError_t launch_mx_quant_rows_gu(const void *wg, const void *wu, int64_t R, int f, uint8_t *codes,
                                    uint8_t *scales, cudaStream_t st, bool tiled) {
  mx_quant_rows_gu_kernel<<<(unsigned)((R + 7) / 8), 256, 0, st>>>(static_cast<const bf16 *>(wg),
                                                                    static_cast<const bf16 *>(wu), R, f, codes,
                                                                    scales, tiled);
  return cudaGetLastError();
}

}  // namespace moe
