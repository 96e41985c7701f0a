// extern "C" entry points of libmoe: argument validation, workspace carve-up, and the
// composition of the layer step.  Every step runs in this library's kernels; nothing
// here touches the host copy of any tensor.
#include <string.h>

#include <initializer_list>

#include "common.cuh"

using namespace moe;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_cfg(const moe_config *c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->d <= 0 || c->f <= 0 || c->E <= 0 || c->k <= 0) return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_BF16 && c->dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
  if (c->prec != MOE_PREC_NATIVE && c->prec != MOE_PREC_MXFP8) return MOE_ERR_INVALID_ARG;
  if (c->E > MAX_E || c->k > MAX_K || c->k > c->E) return MOE_ERR_UNSUPPORTED;
  if (c->d % 128 || c->f % 128) return MOE_ERR_UNSUPPORTED;
  if (c->T * (int64_t)c->k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (c->prec == MOE_PREC_MXFP8 && c->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// All pointers non-null and 16-byte aligned (rows are moved as 16-byte vectors / TMA tiles).
int check_ptrs(std::initializer_list<const void *> ps) {
  for (const void *p : ps)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}
// As check_ptrs, but NULL is allowed (an optional buffer).
int check_ptrs_or_null(std::initializer_list<const void *> ps) {
  for (const void *p : ps)
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}
// Pointers that only need to be non-null and 4-byte aligned (index and fp32 arrays).
int check_ptrs4(std::initializer_list<const void *> ps) {
  for (const void *p : ps)
    if (!p || (reinterpret_cast<uintptr_t>(p) & 3u)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

cudaStream_t S(moe_stream_t s) { return static_cast<cudaStream_t>(s); }

#define RETURN_IF(x)        \
  do {                      \
    int _rc = (x);          \
    if (_rc) return _rc;    \
  } while (0)

}  // namespace

extern "C" {

size_t moe_workspace_size(const moe_config *cfg) {
  if (!cfg || cfg->T < 0 || cfg->E <= 0 || cfg->d <= 0 || cfg->k <= 0) return 0;
  return ws_layout(shape_of(cfg)).total;
}

size_t moe_mx_saved_bytes(const moe_config *cfg) {
  if (!cfg || cfg->T < 0 || cfg->E <= 0 || cfg->d <= 0 || cfg->f <= 0 || cfg->k <= 0) return 0;
  return mx_saved_layout(shape_of(cfg)).total;
}

int moe_get_error(void *ws, moe_stream_t stream, int32_t *code) {
  if (!ws || !code) return MOE_ERR_INVALID_ARG;
  int32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, err_word(ws), sizeof(int32_t), cudaMemcpyDeviceToHost, S(stream));
  if (e == cudaSuccess) e = cudaMemsetAsync(err_word(ws), 0, sizeof(int32_t), S(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(S(stream));
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  *code = h;
  return MOE_OK;
}

int moe_debug_set_gemm_stall_ns(uint64_t ns) {
  if (ns > MOE_DEBUG_STALL_MAX_NS) return MOE_ERR_INVALID_ARG;
  set_gemm_stall_ns(ns);
  return MOE_OK;
}

int moe_route_topk(const moe_config *cfg, const void *x, const void *w_router, const float *bias,
                   float *logits, int32_t *topk_idx, float *topk_gate, void *ws, moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  if (cfg->T == 0) return MOE_OK;
  RETURN_IF(check_ptrs4({x, w_router, topk_idx, topk_gate}));
  if (!ws) return MOE_ERR_WORKSPACE;
  Shape s = shape_of(cfg);
  return cuda_rc(launch_route_topk(s, x, w_router, bias, logits, topk_idx, topk_gate, err_word(ws), S(stream)));
}

int moe_topk_gating(const moe_config *cfg, const float *logits, int32_t *topk_idx, float *topk_gate,
                    void *ws, moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  if (cfg->T == 0) return MOE_OK;
  RETURN_IF(check_ptrs4({logits, topk_idx, topk_gate}));
  if (!ws) return MOE_ERR_WORKSPACE;
  return cuda_rc(launch_topk_gating(shape_of(cfg), logits, topk_idx, topk_gate, err_word(ws), S(stream)));
}

int moe_build_offsets(const moe_config *cfg, const int32_t *topk_idx, int32_t *counts, int32_t *offsets,
                      int32_t *slot_of_pair, int32_t *pair_of_slot, void *ws, moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  RETURN_IF(check_ptrs4({counts, offsets}));
  if (cfg->T > 0) RETURN_IF(check_ptrs4({topk_idx, slot_of_pair, pair_of_slot}));
  if (!ws) return MOE_ERR_WORKSPACE;
  Shape s = shape_of(cfg);
  WsLayout L = ws_layout(s);
  int32_t *bc = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + L.block_counts);
  return cuda_rc(launch_build_offsets(s, topk_idx, counts, offsets, slot_of_pair, pair_of_slot, bc,
                                      err_word(ws), S(stream)));
}

int moe_permute(const moe_config *cfg, const void *x, const int32_t *slot_of_pair, void *x_perm,
                moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  if (cfg->T == 0) return MOE_OK;
  RETURN_IF(check_ptrs({x, x_perm}));
  RETURN_IF(check_ptrs4({slot_of_pair}));
  return cuda_rc(launch_permute(shape_of(cfg), x, slot_of_pair, x_perm, S(stream)));
}

int moe_grouped_swiglu_fwd(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                           const void *w_gate, const void *w_up, const void *w_down, void *hu, void *a,
                           void *y_perm, void *ws, moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  if (cfg->T == 0) return MOE_OK;
  RETURN_IF(check_ptrs({x_perm, w_gate, w_up, w_down, hu, a, y_perm}));
  RETURN_IF(check_ptrs4({offsets}));
  if (!ws) return MOE_ERR_WORKSPACE;
  return launch_grouped_fwd(shape_of(cfg), x_perm, offsets, w_gate, w_up, w_down, hu, a, y_perm, ws,
                            S(stream));
}

int moe_grouped_swiglu_bwd(const moe_config *cfg, const void *dy_perm, const void *x_perm, const void *hu,
                           const void *a, const int32_t *offsets, const void *w_gate, const void *w_up,
                           const void *w_down, void *dhu, void *dx_perm, void *dw_gate, void *dw_up,
                           void *dw_down, void *ws, moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  RETURN_IF(check_ptrs({w_gate, w_up, w_down, dw_gate, dw_up, dw_down}));
  RETURN_IF(check_ptrs4({offsets}));
  if (!ws) return MOE_ERR_WORKSPACE;
  Shape s = shape_of(cfg);
  if (cfg->T == 0) {
    // no routed rows: every expert's weight gradient is zero
    size_t wb = (size_t)s.E * s.d * s.f * s.es();
    cudaError_t e = cudaMemsetAsync(dw_gate, 0, wb, S(stream));
    if (e == cudaSuccess) e = cudaMemsetAsync(dw_up, 0, wb, S(stream));
    if (e == cudaSuccess) e = cudaMemsetAsync(dw_down, 0, wb, S(stream));
    return cuda_rc(e);
  }
  RETURN_IF(check_ptrs({dy_perm, x_perm, hu, a, dhu, dx_perm}));
  return launch_grouped_bwd(s, dy_perm, x_perm, hu, a, offsets, w_gate, w_up, w_down, dhu, dx_perm,
                            dw_gate, dw_up, dw_down, ws, S(stream));
}

int moe_mx_quantize_rows(const void *src, int64_t rows, int32_t cols, const int32_t *offsets, int32_t E,
                         int64_t rows_bound, uint8_t *codes, uint8_t *scales, moe_stream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 32 || (offsets && (cols % 128 || E <= 0 || E > MAX_E)))
    return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (offsets && rows_bound < rows + 127 * (int64_t)E) return MOE_ERR_INVALID_ARG;
  RETURN_IF(check_ptrs({src, codes}));
  RETURN_IF(check_ptrs4({scales}));
  return cuda_rc(launch_mx_quant_rows(src, rows, cols, offsets, E, offsets ? rows_bound : rows, codes, scales,
                                      S(stream)));
}

int moe_permute_mxfp8(const moe_config *cfg, const void *x, const int32_t *slot_of_pair, const int32_t *offsets,
                      void *x_perm, int64_t rows_bound, uint8_t *codes, uint8_t *scales, moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  if (cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (cfg->T == 0) return MOE_OK;
  const Shape s = shape_of(cfg);
  if (rows_bound < s.Ppad()) return MOE_ERR_INVALID_ARG;
  RETURN_IF(check_ptrs({x, x_perm, codes}));
  RETURN_IF(check_ptrs4({slot_of_pair, offsets, scales}));
  return cuda_rc(launch_mx_permute(x, slot_of_pair, offsets, s.E, s.T, s.k, s.d, x_perm, codes, scales, S(stream)));
}

int moe_dispatch_mxfp8(const moe_config *cfg, const void *x, const int32_t *pair_of_slot, const int32_t *offsets,
                       int64_t rows_bound, void *x_perm, uint8_t *codes_r, uint8_t *scales_r, uint8_t *codes_c,
                       uint8_t *scales_c, moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  if (cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (cfg->T == 0) return MOE_OK;
  const Shape s = shape_of(cfg);
  if (rows_bound < s.Ppad()) return MOE_ERR_INVALID_ARG;
  RETURN_IF(check_ptrs({x, codes_r, codes_c}));
  RETURN_IF(check_ptrs_or_null({x_perm}));
  RETURN_IF(check_ptrs4({pair_of_slot, offsets, scales_r, scales_c}));
  return cuda_rc(launch_mx_dispatch(x, pair_of_slot, offsets, s.E, s.k, s.d, rows_bound, x_perm, codes_r, scales_r,
                                    codes_c, scales_c, S(stream), /*tiled=*/false));
}

int moe_combine_bwd_mxfp8(const moe_config *cfg, const void *dy, const void *y_perm, const int32_t *pair_of_slot,
                          const int32_t *offsets, const float *topk_gate, int64_t rows_bound, void *dy_perm,
                          float *dgate, uint8_t *codes_r, uint8_t *scales_r, uint8_t *codes_c, uint8_t *scales_c,
                          moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  if (cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (cfg->T == 0) return MOE_OK;
  const Shape s = shape_of(cfg);
  if (rows_bound < s.Ppad()) return MOE_ERR_INVALID_ARG;
  RETURN_IF(check_ptrs({dy, y_perm, codes_r, codes_c}));
  RETURN_IF(check_ptrs_or_null({dy_perm}));
  RETURN_IF(check_ptrs4({pair_of_slot, offsets, topk_gate, dgate, scales_r, scales_c}));
  return cuda_rc(launch_mx_combine_bwd(dy, y_perm, pair_of_slot, offsets, topk_gate, s.E, s.k, s.d, rows_bound,
                                       dy_perm, dgate, codes_r, scales_r, codes_c, scales_c, S(stream),
                                       /*tiled=*/false));
}

int moe_mx_quantize_cols(const void *src, int64_t rows, int32_t cols, const int32_t *offsets, int32_t E,
                         int64_t rows_bound, uint8_t *codes, uint8_t *scales, moe_stream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 32 || (offsets && (E <= 0 || E > MAX_E))) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (offsets && rows_bound < rows + 127 * (int64_t)E) return MOE_ERR_INVALID_ARG;
  RETURN_IF(check_ptrs({src, codes}));
  RETURN_IF(check_ptrs4({scales}));
  return cuda_rc(launch_mx_quant_cols(src, rows, cols, offsets, E, offsets ? rows_bound : rows, codes, scales,
                                      S(stream)));
}

int moe_unpermute_combine(const moe_config *cfg, const void *y_perm, const int32_t *slot_of_pair,
                          const float *topk_gate, void *y, moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  if (cfg->T == 0) return MOE_OK;
  RETURN_IF(check_ptrs({y_perm, y}));
  RETURN_IF(check_ptrs4({slot_of_pair, topk_gate}));
  return cuda_rc(launch_unpermute_combine(shape_of(cfg), y_perm, slot_of_pair, topk_gate, y, S(stream)));
}

int moe_combine_bwd(const moe_config *cfg, const void *dy, const void *y_perm, const int32_t *slot_of_pair,
                    const float *topk_gate, void *dy_perm, float *dgate, moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  if (cfg->T == 0) return MOE_OK;
  RETURN_IF(check_ptrs({dy, y_perm, dy_perm}));
  RETURN_IF(check_ptrs4({slot_of_pair, topk_gate, dgate}));
  return cuda_rc(launch_combine_bwd(shape_of(cfg), dy, y_perm, slot_of_pair, topk_gate, dy_perm, dgate,
                                    S(stream)));
}

int moe_unpermute_sum(const moe_config *cfg, const void *dx_perm, const int32_t *slot_of_pair, void *dx,
                      moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  if (cfg->T == 0) return MOE_OK;
  RETURN_IF(check_ptrs({dx_perm, dx}));
  RETURN_IF(check_ptrs4({slot_of_pair}));
  return cuda_rc(launch_unpermute_sum(shape_of(cfg), dx_perm, slot_of_pair, nullptr, nullptr, nullptr,
                                      nullptr, false, dx, S(stream)));
}

int moe_route_bwd(const moe_config *cfg, const float *dgate, const float *topk_gate, const int32_t *topk_idx,
                  const void *x, const void *w_router, void *dx, float *dw_router, void *ws,
                  moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  RETURN_IF(check_ptrs4({w_router, dw_router}));
  if (!ws) return MOE_ERR_WORKSPACE;
  Shape s = shape_of(cfg);
  if (cfg->T > 0) {
    RETURN_IF(check_ptrs4({dgate, topk_gate, topk_idx}));
    RETURN_IF(check_ptrs({x, dx}));
  }
  WsLayout L = ws_layout(s);
  char *w = static_cast<char *>(ws);
  void *w_rt = w + L.w_rt;
  float *part = reinterpret_cast<float *>(w + L.dwr_partial);
  RETURN_IF(cuda_rc(launch_router_transpose(s, w_router, w_rt, S(stream))));
  RETURN_IF(cuda_rc(launch_router_wgrad(s, dgate, topk_gate, topk_idx, x, part, dw_router, S(stream))));
  return cuda_rc(launch_unpermute_sum(s, nullptr, nullptr, dgate, topk_gate, topk_idx, w_rt, true, dx,
                                      S(stream)));
}

// The shared expert as a problem of its own: one group (E = 1) of all T tokens (k = 1).
static Shape shared_shape(const Shape &s) {
  Shape t = s;
  t.E = 1;
  t.k = 1;
  return t;
}

// 0: no shared expert; 1: a complete one; -1: some of its pointers missing.
static int shared_expert(const moe_layer_weights *w) {
  const int n = (w->w_shared_gate != nullptr) + (w->w_shared_up != nullptr) + (w->w_shared_down != nullptr);
  return n == 0 ? 0 : n == 3 ? 1 : -1;
}

static int layer_fwd_common(const moe_config *cfg, const moe_layer_weights *w, const void *x, void *y,
                            const moe_layer_saved *sv, void *ws, moe_stream_t stream, bool route) {
  RETURN_IF(check_cfg(cfg));
  if (!w || !sv) return MOE_ERR_INVALID_ARG;
  if (!ws) return MOE_ERR_WORKSPACE;
  Shape s = shape_of(cfg);
  const int shared = shared_expert(w);
  if (shared < 0) return MOE_ERR_INVALID_ARG;
  RETURN_IF(check_ptrs({w->w_gate, w->w_up, w->w_down}));
  RETURN_IF(check_ptrs4({sv->counts, sv->offsets}));
  if (route) RETURN_IF(check_ptrs4({w->w_router}));
  if (shared) RETURN_IF(check_ptrs({w->w_shared_gate, w->w_shared_up, w->w_shared_down}));
  const bool mx = s.prec == MOE_PREC_MXFP8;
  if (mx) RETURN_IF(check_ptrs_or_null({sv->mx_saved}));
  // MXFP8 with the saved copies: the routed rows move as E4M3 only and x_perm is unused
  const bool rows_fp8 = mx && sv->mx_saved;
  if (cfg->T > 0) {
    RETURN_IF(check_ptrs({x, y, sv->a, sv->y_perm}));
    RETURN_IF(rows_fp8 ? check_ptrs_or_null({sv->x_perm}) : check_ptrs({sv->x_perm}));
    RETURN_IF(check_ptrs_or_null({sv->hu}));
    RETURN_IF(check_ptrs4({sv->topk_idx, sv->topk_gate, sv->slot_of_pair, sv->pair_of_slot}));
    if (shared) {
      RETURN_IF(check_ptrs({sv->shared_a}));
      RETURN_IF(check_ptrs_or_null({sv->shared_hu}));
    }
  }
  cudaStream_t st = S(stream);
  int *err = err_word(ws);
  WsLayout L = ws_layout(s);
  int32_t *bc = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + L.block_counts);
  if (route && cfg->T > 0)
    RETURN_IF(cuda_rc(launch_route_topk(s, x, w->w_router, w->bias, sv->logits, sv->topk_idx, sv->topk_gate,
                                        err, st)));
  RETURN_IF(cuda_rc(launch_build_offsets(s, sv->topk_idx, sv->counts, sv->offsets, sv->slot_of_pair,
                                         sv->pair_of_slot, bc, err, st)));
  if (cfg->T == 0) return MOE_OK;
  uint8_t *mxs = mx ? static_cast<uint8_t *>(sv->mx_saved) : nullptr;
  if (mx) {
    const int64_t R = s.Ppad();
    if (mxs) {
      // FP8 dispatch: each routed row of x is read once and written only in MXFP8, along d
      // for the forward GEMM and down the token axis for the backward's weight gradient
      const MxSavedLayout M = mx_saved_layout(s);
      uint8_t *xqr = mxs + M.xq_r, *xqt = mxs + M.xq_t;
      RETURN_IF(cuda_rc(launch_mx_dispatch(x, sv->pair_of_slot, sv->offsets, s.E, s.k, s.d, R, nullptr, xqr,
                                           xqr + R * s.d, xqt, xqt + R * s.d, st)));
    } else {
      // the permute also writes x_perm's MXFP8 rows where the forward GEMM reads them
      uint8_t *xq = static_cast<uint8_t *>(ws) + L.xq_r;
      RETURN_IF(cuda_rc(launch_mx_permute(x, sv->slot_of_pair, sv->offsets, s.E, s.T, s.k, s.d, sv->x_perm, xq,
                                          xq + R * s.d, st, /*tiled=*/true)));
    }
  } else {
    RETURN_IF(cuda_rc(launch_permute(s, x, sv->slot_of_pair, sv->x_perm, st)));
  }
  RETURN_IF(launch_grouped_fwd(s, sv->x_perm, sv->offsets, w->w_gate, w->w_up, w->w_down, sv->hu, sv->a,
                               sv->y_perm, ws, st, mx, mxs, /*wfill=*/true));
  if (shared) {
    // the shared expert's output goes straight into y; the combine then adds to it
    int32_t *go = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + L.group_offsets);
    RETURN_IF(cuda_rc(launch_group_offsets(go, s.T, st)));
    RETURN_IF(launch_grouped_fwd(shared_shape(s), x, go, w->w_shared_gate, w->w_shared_up, w->w_shared_down,
                                 sv->shared_hu, sv->shared_a, y, ws, st));
  }
  return cuda_rc(launch_unpermute_combine(s, sv->y_perm, sv->slot_of_pair, sv->topk_gate, y, st, shared));
}

int moe_layer_fwd(const moe_config *cfg, const moe_layer_weights *w, const void *x, void *y,
                  const moe_layer_saved *saved, void *ws, moe_stream_t stream) {
  return layer_fwd_common(cfg, w, x, y, saved, ws, stream, true);
}

int moe_layer_fwd_routed(const moe_config *cfg, const moe_layer_weights *w, const void *x, void *y,
                         const moe_layer_saved *saved, void *ws, moe_stream_t stream) {
  return layer_fwd_common(cfg, w, x, y, saved, ws, stream, false);
}

int moe_layer_bwd(const moe_config *cfg, const moe_layer_weights *w, const void *x, const void *dy,
                  const moe_layer_saved *sv, const moe_layer_grads *g, void *ws, moe_stream_t stream) {
  RETURN_IF(check_cfg(cfg));
  if (!w || !sv || !g) return MOE_ERR_INVALID_ARG;
  if (!ws) return MOE_ERR_WORKSPACE;
  Shape s = shape_of(cfg);
  cudaStream_t st = S(stream);
  int *err = err_word(ws);
  const bool router = g->dw_router != nullptr;
  const int shared = shared_expert(w);
  if (shared < 0) return MOE_ERR_INVALID_ARG;
  RETURN_IF(check_ptrs({w->w_gate, w->w_up, w->w_down, g->dw_gate, g->dw_up, g->dw_down}));
  RETURN_IF(check_ptrs4({sv->offsets}));
  if (router) RETURN_IF(check_ptrs4({w->w_router, g->dw_router}));
  if ((router || s.prec == MOE_PREC_MXFP8) && cfg->T > 0) RETURN_IF(check_ptrs4({sv->pair_of_slot}));
  const bool mx = s.prec == MOE_PREC_MXFP8;
  // MXFP8: dy_perm moves in MXFP8 only; with the saved copies x_perm is unused too
  const bool rows_fp8 = mx && sv->mx_saved;
  if (shared)
    RETURN_IF(check_ptrs({w->w_shared_gate, w->w_shared_up, w->w_shared_down, g->dw_shared_gate,
                          g->dw_shared_up, g->dw_shared_down}));
  if (s.prec == MOE_PREC_MXFP8) RETURN_IF(check_ptrs_or_null({sv->mx_saved}));
  if (cfg->T > 0) {
    RETURN_IF(check_ptrs({x, dy, g->dx, sv->a, sv->y_perm, g->dhu, g->dx_perm}));
    RETURN_IF(rows_fp8 ? check_ptrs_or_null({sv->x_perm}) : check_ptrs({sv->x_perm}));
    RETURN_IF(mx ? check_ptrs_or_null({g->dy_perm}) : check_ptrs({g->dy_perm}));
    RETURN_IF(check_ptrs_or_null({sv->hu}));
    RETURN_IF(check_ptrs4({sv->topk_idx, sv->topk_gate, sv->slot_of_pair, g->dgate}));
    if (shared) {
      RETURN_IF(check_ptrs({sv->shared_a, g->shared_dhu}));
      RETURN_IF(check_ptrs_or_null({sv->shared_hu}));
    }
  }
  if (cfg->T == 0) {
    size_t wb = (size_t)s.E * s.d * s.f * s.es();
    cudaError_t e = cudaMemsetAsync(g->dw_gate, 0, wb, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(g->dw_up, 0, wb, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(g->dw_down, 0, wb, st);
    if (e == cudaSuccess && router) e = cudaMemsetAsync(g->dw_router, 0, (size_t)s.d * s.E * 4, st);
    const size_t sb = (size_t)s.d * s.f * s.es();
    if (e == cudaSuccess && shared) e = cudaMemsetAsync(g->dw_shared_gate, 0, sb, st);
    if (e == cudaSuccess && shared) e = cudaMemsetAsync(g->dw_shared_up, 0, sb, st);
    if (e == cudaSuccess && shared) e = cudaMemsetAsync(g->dw_shared_down, 0, sb, st);
    return cuda_rc(e);
  }
  if (mx) {
    // FP8 dispatch of the backward: dy_perm exists only as the MXFP8 copies both
    // down-projection GEMMs read, written by the combine's backward itself
    const WsLayout L = ws_layout(s);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    const int64_t R = s.Ppad();
    uint8_t *dyq = w8 + L.dyq_r, *dyqt = w8 + L.dyq_t;
    RETURN_IF(cuda_rc(launch_mx_combine_bwd(dy, sv->y_perm, sv->pair_of_slot, sv->offsets, sv->topk_gate, s.E, s.k,
                                            s.d, R, nullptr, g->dgate, dyq, dyq + R * s.d, dyqt, dyqt + R * s.d,
                                            st)));
  } else {
    RETURN_IF(cuda_rc(launch_combine_bwd(s, dy, sv->y_perm, sv->slot_of_pair, sv->topk_gate, g->dy_perm,
                                         g->dgate, st)));
  }
  // recompute: [h | u] = x_perm [Wg | Wu] into dhu, where the SwiGLU backward then runs in place
  uint8_t *mxs = mx ? static_cast<uint8_t *>(sv->mx_saved) : nullptr;
  const void *hu = sv->hu;
  if (!hu) {
    // with the saved copies the forward's MXFP8 rows of x_perm are read again as they are
    RETURN_IF(launch_grouped_fwd(s, sv->x_perm, sv->offsets, w->w_gate, w->w_up, w->w_down, g->dhu, nullptr,
                                 nullptr, ws, st, /*x_quantized=*/rows_fp8, mxs, /*wfill=*/false));
    hu = g->dhu;
  }
  // MXFP8: [dh | du] is kept in MXFP8 only (g->dhu serves as the recompute's scratch)
  RETURN_IF(launch_grouped_bwd(s, g->dy_perm, sv->x_perm, hu, sv->a, sv->offsets, w->w_gate, w->w_up,
                               w->w_down, g->dhu, g->dx_perm, g->dw_gate, g->dw_up, g->dw_down, ws, st, mxs, mx,
                               /*keep_dhu=*/!mx));
  if (shared) {
    // one group of all tokens: its dy is dY itself (weight 1) and its dx, in token order,
    // is written to dx, to which the routed experts' rows are then added
    const Shape s1 = shared_shape(s);
    WsLayout L = ws_layout(s);
    int32_t *go = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + L.group_offsets);
    RETURN_IF(cuda_rc(launch_group_offsets(go, s.T, st)));
    const void *shu = sv->shared_hu;
    if (!shu) {
      RETURN_IF(launch_grouped_fwd(s1, x, go, w->w_shared_gate, w->w_shared_up, w->w_shared_down, g->shared_dhu,
                                   nullptr, nullptr, ws, st));
      shu = g->shared_dhu;
    }
    RETURN_IF(launch_grouped_bwd(s1, dy, x, shu, sv->shared_a, go, w->w_shared_gate, w->w_shared_up,
                                 w->w_shared_down, g->shared_dhu, g->dx, g->dw_shared_gate, g->dw_shared_up,
                                 g->dw_shared_down, ws, st));
  }
  if (!router)
    return cuda_rc(launch_unpermute_sum(s, g->dx_perm, sv->slot_of_pair, nullptr, nullptr, nullptr, nullptr,
                                        shared, g->dx, st));
  WsLayout L = ws_layout(s);
  char *wsc = static_cast<char *>(ws);
  void *w_rt = wsc + L.w_rt;
  RETURN_IF(cuda_rc(launch_router_transpose(s, w->w_router, w_rt, st)));
  // dW_r = x^T dz over the routed rows: x_perm's rows, or x's rows through pair_of_slot
  RETURN_IF(cuda_rc(launch_router_wgrad_grouped(s, sv->x_perm, sv->pair_of_slot, sv->offsets, g->dgate,
                                                sv->topk_gate, reinterpret_cast<float *>(wsc + L.dz_slot),
                                                reinterpret_cast<float *>(wsc + L.rg_partial), g->dw_router,
                                                st, rows_fp8 ? x : nullptr)));
  // dx = sum_j dx_perm[slot(t,j)] + dz W_r^T in one pass
  return cuda_rc(launch_unpermute_sum(s, g->dx_perm, sv->slot_of_pair, g->dgate, sv->topk_gate, sv->topk_idx,
                                      w_rt, shared, g->dx, st));
}

}  // extern "C"
