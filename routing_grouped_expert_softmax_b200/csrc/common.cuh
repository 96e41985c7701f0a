// Shared helpers for libmoe's kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

typedef __nv_bfloat16 bf16;

// Layout of the small fixed part of the workspace (bytes).
constexpr size_t WS_ERR = 0;          // int32 device error word
constexpr size_t WS_FIXED = 256;      // everything else starts here

constexpr int MAX_E = 256;
constexpr int MAX_K = 8;
constexpr int SCATTER_CHUNK = 1024;   // routed pairs per block in the metadata kernels

struct Shape {
  int64_t T;
  int d, E, k, f;
  int dtype;
  int prec = MOE_PREC_NATIVE;
  // rows of an expert buffer padded to 128 rows per expert (MXFP8 operands), upper bound
  int64_t Ppad() const { return P() + 127 * (int64_t)E; }
  int64_t P() const { return T * (int64_t)k; }
  int es() const { return dtype == MOE_BF16 ? 2 : 4; }
};

inline Shape shape_of(const moe_config *c) {
  Shape s;
  s.T = c->T; s.d = c->d; s.E = c->E; s.k = c->k; s.f = c->f; s.dtype = c->dtype; s.prec = c->prec;
  return s;
}

inline int *err_word(void *ws) { return reinterpret_cast<int *>(static_cast<char *>(ws) + WS_ERR); }

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace carve-up shared by the host launchers.
struct WsLayout {
  size_t block_counts;   // int32 [nblocks][E]
  size_t w_rt;           // [E][d] in the storage type (transposed router weight)
  size_t dwr_partial;    // fp32 [RB_SPLIT][E][d]
  size_t wt;             // fp32 storage only: Wg^T, Wu^T [E][f][d] and Wd^T [E][d][f]
  size_t dz_slot;        // fp32 [P]: router logit gradient of the pair in each slot
  size_t rg_partial;     // fp32 [P/64 + E][d]: per-chunk router weight-gradient sums
  // MXFP8 operands (codes, then scales), present when prec == MOE_PREC_MXFP8:
  //   *_r: blocks along the row (K-major use), *_t: blocks down the rows (token axis)
  size_t xq_r, aq_r, dyq_r, dhuq_r, xq_t, aq_t, dyq_t, dhuq_t;  // activations, Ppad rows
  size_t wgu_c, wd_c, wd_r, wgu_r;                              // weights
  // bf16 weight-gradient GEMMs: every expert's last partial K-block of their two operands,
  // [E * 64][C] each (rows past the expert zero), C up to max(d, f) and max(d, 2f)
  size_t wg_tail_a, wg_tail_b;
  // int32 {0, T}: the shared expert's single group.  Last, so that a layout for the shared
  // expert's shape (E = 1, k = 1: every region no larger) never reaches it.
  size_t group_offsets;
  size_t total;
};
// bytes of an MXFP8 operand [rows][cols] with scales along the row / down the rows
inline size_t mx_bytes_r(int64_t rows, int64_t cols) { return align_up((size_t)(rows * cols + rows * (cols / 32)), 256); }
// (token-axis scales in the GEMMs' tile layout cover the rows rounded up to 128)
inline size_t mx_bytes_t(int64_t rows, int64_t cols) {
  return align_up((size_t)(rows * cols + ((rows + 127) / 128) * 4 * cols), 256);
}
constexpr int RB_SPLIT = 16;          // token splits of the router weight-gradient reduction
constexpr int WGRAD_TAIL_ROWS = 64;   // rows of a bf16 weight-gradient K-block (one tail per expert)


inline WsLayout ws_layout(const Shape &s) {
  WsLayout L;
  size_t off = WS_FIXED;
  int64_t nb = (s.P() + SCATTER_CHUNK - 1) / SCATTER_CHUNK;
  L.block_counts = off; off = align_up(off + (size_t)nb * s.E * 4, 256);
  L.w_rt = off;         off = align_up(off + (size_t)s.E * s.d * 4, 256);
  L.dwr_partial = off;  off = align_up(off + (size_t)RB_SPLIT * s.E * s.d * 4, 256);
  L.wt = off;
  if (s.dtype == MOE_F32) off = align_up(off + (size_t)3 * s.E * s.d * s.f * 4, 256);
  L.dz_slot = off;      off = align_up(off + (size_t)s.P() * 4, 256);
  L.rg_partial = off;   off = align_up(off + (size_t)((s.P() + 63) / 64 + s.E) * s.d * 4, 256);
  L.xq_r = L.aq_r = L.dyq_r = L.dhuq_r = L.xq_t = L.aq_t = L.dyq_t = L.dhuq_t = 0;
  L.wgu_c = L.wd_c = L.wd_r = L.wgu_r = 0;
  if (s.prec == MOE_PREC_MXFP8) {
    const int64_t R = s.Ppad(), ed = (int64_t)s.E * s.d, ef = (int64_t)s.E * s.f;
    L.xq_r = off;   off += mx_bytes_r(R, s.d);
    L.aq_r = off;   off += mx_bytes_r(R, s.f);
    L.dyq_r = off;  off += mx_bytes_r(R, s.d);
    L.dhuq_r = off; off += mx_bytes_r(R, 2 * s.f);
    L.xq_t = off;   off += mx_bytes_t(R, s.d);
    L.aq_t = off;   off += mx_bytes_t(R, s.f);
    L.dyq_t = off;  off += mx_bytes_t(R, s.d);
    L.dhuq_t = off; off += mx_bytes_t(R, 2 * s.f);
    L.wgu_c = off;  off += mx_bytes_t(ed, 2 * s.f);
    L.wd_c = off;   off += mx_bytes_t(ef, s.d);
    L.wd_r = off;   off += mx_bytes_r(ef, s.d);
    L.wgu_r = off;  off += mx_bytes_r(ed, 2 * s.f);
  }
  L.wg_tail_a = L.wg_tail_b = 0;
  if (s.dtype == MOE_BF16 && s.prec == MOE_PREC_NATIVE) {
    const size_t rows = (size_t)s.E * WGRAD_TAIL_ROWS;
    L.wg_tail_a = off; off = align_up(off + rows * (size_t)(s.d > s.f ? s.d : s.f) * 2, 256);
    L.wg_tail_b = off; off = align_up(off + rows * (size_t)(s.d > 2 * s.f ? s.d : 2 * s.f) * 2, 256);
  }
  L.group_offsets = off; off += 256;   // {0, T}: the shared expert's single group
  L.total = off;
  return L;
}

// Layout of moe_layer_saved.mx_saved: the routed experts' weights in MXFP8 in the four
// orientations the grouped GEMMs read, the permuted layer input in MXFP8 along d and down the
// expert-padded token axis, and the activation a down the token axis (the weight-gradient
// GEMMs' operands), each as codes then scales in the GEMMs' tile layout.
struct MxSavedLayout {
  size_t wgu_c, wd_c, wd_r, wgu_r;   // as the workspace's regions of the same names
  size_t xq_r, xq_t, aq_t;           // [Ppad][d] along d, [Ppad][d] and [Ppad][f] along tokens
  size_t total;
};
inline MxSavedLayout mx_saved_layout(const Shape &s) {
  MxSavedLayout L{};
  if (s.prec != MOE_PREC_MXFP8) return L;
  const int64_t ed = (int64_t)s.E * s.d, ef = (int64_t)s.E * s.f, R = s.Ppad();
  size_t off = 0;
  L.wgu_c = off; off += mx_bytes_t(ed, 2 * s.f);
  L.wd_c = off;  off += mx_bytes_t(ef, s.d);
  L.wd_r = off;  off += mx_bytes_r(ef, s.d);
  L.wgu_r = off; off += mx_bytes_r(ed, 2 * s.f);
  L.xq_r = off;  off += mx_bytes_r(R, s.d);
  L.xq_t = off;  off += mx_bytes_t(R, s.d);
  L.aq_t = off;  off += mx_bytes_t(R, s.f);
  L.total = off;
  return L;
}

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// 16-byte vector <-> fp32 lanes.  A uint4 holds 8 bf16 or 4 fp32.
template <typename T> struct Vec;
template <> struct Vec<bf16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const uint4 &v, float *o) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) { float2 f = __bfloat1622float2(h[i]); o[2 * i] = f.x; o[2 * i + 1] = f.y; }
  }
  __device__ __forceinline__ static uint4 store(const float *o) {
    uint4 v;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
    return v;
  }
};
template <> struct Vec<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const uint4 &v, float *o) {
    o[0] = __uint_as_float(v.x); o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z); o[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static uint4 store(const float *o) {
    return make_uint4(__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]),
                      __float_as_uint(o[3]));
  }
};

__device__ __forceinline__ void set_error(int *err, int bit) {
  if (err) atomicOr(err, bit);
}

// Failure-detection test hook of the grouped GEMMs (grouped_gemm.cu): ns > 0 makes every later
// single-CTA launch wait up to ns on a barrier nothing arrives on and take its abort path.
void set_gemm_stall_ns(uint64_t ns);

// ---- internal launchers (host side), implemented in routing.cu / rowops.cu / grouped_gemm.cu
cudaError_t launch_route_topk(const Shape &s, const void *x, const void *w_r, const float *bias,
                              float *logits, int32_t *idx, float *gate, int *err, cudaStream_t st);
// tensor-core router (bf16, E % 8 == 0) with the top-k fused into its epilogue
int launch_router_tc(const Shape &s, const void *x, const void *w_r, const float *bias, float *logits,
                     int32_t *idx, float *gate, int *err, cudaStream_t st);
cudaError_t launch_topk_gating(const Shape &s, const float *logits, int32_t *idx, float *gate,
                               int *err, cudaStream_t st);
cudaError_t launch_build_offsets(const Shape &s, const int32_t *idx, int32_t *counts,
                                 int32_t *offsets, int32_t *slot_of_pair, int32_t *pair_of_slot,
                                 int32_t *block_counts, int *err, cudaStream_t st);
cudaError_t launch_permute(const Shape &s, const void *x, const int32_t *slot_of_pair,
                           void *x_perm, cudaStream_t st);
// accumulate: add to the values y already holds (the shared expert's output)
cudaError_t launch_unpermute_combine(const Shape &s, const void *y_perm, const int32_t *sop,
                                     const float *gate, void *y, cudaStream_t st, bool accumulate = false);
cudaError_t launch_group_offsets(int32_t *o, int64_t T, cudaStream_t st);
// FP8 dispatch: the permute that also writes each routed row in MXFP8 (blocks of 32 along d)
// into the expert buffers padded to 128 rows (bf16 storage, d % 32 == 0)
// tiled: scales in the block-scaled GEMMs' tile layout (quant.cu) instead of the plain one
cudaError_t launch_mx_permute(const void *x, const int32_t *sop, const int32_t *offsets, int E, int64_t T, int k,
                              int d, void *x_perm, uint8_t *codes, uint8_t *scales, cudaStream_t st,
                              bool tiled = false);
// The combine's backward for the MXFP8 layer (bf16 storage, d % 128 == 0): dy_perm, dgate as
// launch_combine_bwd, and dy_perm in MXFP8 along d (codes_r) and down the expert-padded token
// axis (codes_c), scales in the GEMMs' tile layout; pos = pair_of_slot; rows_bound = Ppad.
// dy_perm may be null (the bf16 rows are not written); tiled: scales in the GEMMs' tile layout,
// else plain ([rows][d/32] along d, [rows/32][d] down the token axis).
cudaError_t launch_mx_combine_bwd(const void *dy, const void *y_perm, const int32_t *pos, const int32_t *offsets,
                                  const float *gate, int E, int k, int d, int64_t rows_bound, void *dy_perm,
                                  float *dgate, uint8_t *codes_r, uint8_t *scales_r, uint8_t *codes_c,
                                  uint8_t *scales_c, cudaStream_t st, bool tiled = true);
// FP8 dispatch, slot-major: x_perm (a bit copy of each routed row) and x_perm in MXFP8 along d
// (codes_r) and down the expert-padded token axis (codes_c), scales in the GEMMs' tile layout.
// x_perm may be null (the bf16 rows are not written); tiled as for launch_mx_combine_bwd.
cudaError_t launch_mx_dispatch(const void *x, const int32_t *pos, const int32_t *offsets, int E, int k, int d,
                               int64_t rows_bound, void *x_perm, uint8_t *codes_r, uint8_t *scales_r,
                               uint8_t *codes_c, uint8_t *scales_c, cudaStream_t st, bool tiled = true);
cudaError_t launch_combine_bwd(const Shape &s, const void *dy, const void *y_perm,
                               const int32_t *sop, const float *gate, void *dy_perm,
                               float *dgate, cudaStream_t st);
// dx[t] = sum_j dx_perm[slot(t,j)] (+ sum_j dz_j W_r^T[e_j] when w_rt != nullptr)
cudaError_t launch_unpermute_sum(const Shape &s, const void *dx_perm, const int32_t *sop,
                                 const float *dgate, const float *gate, const int32_t *idx,
                                 const void *w_rt, bool accumulate, void *dx, cudaStream_t st);
cudaError_t launch_router_transpose(const Shape &s, const void *w_r, void *w_rt, cudaStream_t st);
// Multiprocessors of the current device (cached per device; 148 if the query fails).
int device_sm_count();

// dW_r from the expert-contiguous rows x_perm and the slot maps (layer backward); x != nullptr:
// the rows are read from the layer input instead, x[pos[slot] / k] (no x_perm kept)
cudaError_t launch_router_wgrad_grouped(const Shape &s, const void *x_perm, const int32_t *pos,
                                        const int32_t *offsets, const float *dgate, const float *gate,
                                        float *dz_slot, float *partial, float *dw_r, cudaStream_t st,
                                        const void *x = nullptr);
cudaError_t launch_router_wgrad(const Shape &s, const float *dgate, const float *gate,
                                const int32_t *idx, const void *x, float *partial,
                                float *dw_r, cudaStream_t st);
// bf16 weight gradients: tails[e*64 + i] = src[offsets[e] + 64*(count_e/64) + i] for
// i < count_e % 64 and zeros for the rest of the expert's 64 rows (src [P][C] bf16); experts
// whose count is a multiple of 64 are left alone (they have no partial K-block).
cudaError_t launch_wgrad_tails(const void *src_a, int C_a, void *tails_a, const void *src_b, int C_b, void *tails_b,
                               const int32_t *offsets, int E, cudaStream_t st);
// MXFP8 only:
//   x_quantized: the workspace already holds x_perm's MXFP8 rows, written by
//     launch_mx_permute into the layout ws_layout(s) gives them;
//   wsaved (layout mx_saved_layout(s)) or nullptr: the weights' MXFP8 copies; wfill: the
//     forward writes all four orientations there (else it reads the ones it needs).
int launch_grouped_fwd(const Shape &s, const void *x_perm, const int32_t *offsets,
                       const void *w_gate, const void *w_up, const void *w_down, void *hu,
                       void *a, void *y_perm, void *ws, cudaStream_t st, bool x_quantized = false,
                       uint8_t *wsaved = nullptr, bool wfill = false);
// dst[b][c][r] = src[b][r][c] (fp32)
cudaError_t launch_transpose_batched(const float *src, float *dst, int B, int R, int C, cudaStream_t st);
// MXFP8 quantisers (quant.cu).  offsets != nullptr: source rows are expert groups written
// into buffers padded to 128 rows per expert (rows_bound: rows the buffer holds).
// tiled: scales in the tile layout the block-scaled GEMMs read (needs K % 128 == 0 along rows).
cudaError_t launch_mx_quant_rows(const void *src, int64_t R, int K, const int32_t *offsets, int E, int64_t rows_bound,
                                 uint8_t *codes, uint8_t *scales, cudaStream_t st, bool tiled = false);
cudaError_t launch_mx_quant_cols(const void *src, int64_t R, int C, const int32_t *offsets, int E, int64_t rows_bound,
                                 uint8_t *codes, uint8_t *scales, cudaStream_t st, bool tiled = false);
cudaError_t launch_mx_quant_cols_gu(const void *wg, const void *wu, int64_t R, int f, uint8_t *codes,
                                    uint8_t *scales, cudaStream_t st, bool tiled = false);
cudaError_t launch_mx_quant_rows_gu(const void *wg, const void *wu, int64_t R, int f, uint8_t *codes,
                                    uint8_t *scales, cudaStream_t st, bool tiled = false);
// Expert weights in both MXFP8 orientations from one read, scales in the tile layout:
// gu: (w0, w1) = (W_gate, W_up) [R = E*d][C = f] -> codes_c [R][2f] (blocks down the rows, gate
// and up interleaved in 64-column chunks) and codes_r [R][2f] (row r = [W_gate[r] | W_up[r]],
// blocks along it); else w0 = W_down [R = E*f][C = d] -> codes_c, codes_r [R][C].  R % 128 == 0,
// C % 128 == 0.
cudaError_t launch_mx_quant_weights(const void *w0, const void *w1, int64_t R, int C, bool gu, uint8_t *codes_c,
                                    uint8_t *scales_c, uint8_t *codes_r, uint8_t *scales_r, cudaStream_t st);
// MXFP8 only:
//   wsaved: the weights' MXFP8 copies a forward wrote (layout mx_saved_layout(s)), read
//     instead of quantising the weights again; nullptr: quantised here, in the workspace;
//   dy_quantized: the workspace already holds dy_perm's MXFP8 copies in both orientations
//     (written by launch_mx_combine_bwd into the layout ws_layout(s) gives them).
int launch_grouped_bwd(const Shape &s, const void *dy_perm, const void *x_perm, const void *hu,
                       const void *a, const int32_t *offsets, const void *w_gate,
                       const void *w_up, const void *w_down, void *dhu, void *dx_perm,
                       void *dw_gate, void *dw_up, void *dw_down, void *ws, cudaStream_t st,
                       const uint8_t *wsaved = nullptr, bool dy_quantized = false, bool keep_dhu = true);

}  // namespace moe
