/*
 * moe.h -- C ABI of libmoe, a single-GPU MoE layer step for NVIDIA B200 (sm_100a).
 *
 * The step, forward and backward, as described in prose by the pages on Ai2's
 * Olmo-core 3 training stack:
 *   unite.ai, "Ai2 κυκλοφορεί το Olmo-Core 3, ανοιχτό σύνολο εκπαίδευσης για MoE
 *     τρισεκατομμυρίων παραμέτρων", section "Παραλληλισμός, Ακρίβεια και Τεχνικές
 *     Μνήμης" (parallelism, precision and memory techniques): routed rows are
 *     written straight into the experts' input buffers; routing metadata stays on
 *     the GPU so the CPU can queue work without waiting for a copy back; a grouped
 *     GEMM runs the experts' many small matmuls together; MXFP8 for selected ops;
 *   ettayeb.fr, "Olmo-core 3 ouvre l'entraînement des MoE à l'échelle du trillion
 *     de paramètres", section "Trois parallélismes, trois optimisations de routage"
 *     (the same three routing optimisations);
 *   qidao123.com, "Ai2开源Olmo-core 3 ...", section "新闻原文": 8 -> 128 experts with
 *     4 selected per token.
 * The pages give no formulas.  This library computes: softmax router with top-k
 * on the logits (ties to the lower expert index), gates renormalised over the k
 * selected experts, a stable counting sort of the routed pairs by expert, a
 * SwiGLU expert FFN y = (silu(x Wg) * (x Wu)) Wd without biases, and the
 * gate-weighted sum of each token's k expert outputs.
 *
 * Conventions for every call
 *   - Every pointer argument is a DEVICE pointer, allocated and owned by the
 *     caller.  The library allocates nothing and keeps no pointer after a call.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and never synchronises the host, except moe_get_error.
 *   - Row-major everywhere.  T tokens, d = model width, E experts, k experts per
 *     token, f = expert FFN width, P = T*k routed pairs.  Pair i = t*k + j is
 *     token t's j-th choice.
 *   - Activations and weights have the element type cfg->dtype (MOE_BF16 or
 *     MOE_F32).  Logits, gates and router gradients are always fp32; indices,
 *     counts, offsets and slots int32.
 *   - Return value: MOE_OK, or a host-detected error (invalid or unsupported
 *     argument, CUDA launch failure); nothing is launched on a host error.
 *     Errors found on the device (an expert index out of range, a timed-out
 *     wait) are OR-ed into an error word inside the workspace and read back by
 *     moe_get_error.
 *   - Supported shapes: 1 <= E <= 256, 1 <= k <= min(E, 8), d and f multiples
 *     of 128, T*k < 2^31.  T = 0 is valid and launches nothing.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef void *moe_stream_t; /* a cudaStream_t */

enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum */
  MOE_ERR_UNSUPPORTED = 2,   /* shape outside the supported set above */
  MOE_ERR_WORKSPACE = 3,     /* workspace pointer missing */
  MOE_ERR_CUDA = 4,          /* a CUDA call failed (launch, tensor map) */
  /* device-side error bits, reported by moe_get_error (OR-ed together): */
  MOE_ERR_DEVICE_INDEX = 16, /* an expert index outside [0, E) */
  MOE_ERR_DEVICE_TIMEOUT = 32, /* a bounded wait inside a kernel gave up */
  MOE_ERR_DEVICE_NAN = 64    /* a NaN router logit (its top-k is undefined) */
};

enum moe_dtype { MOE_F32 = 0, MOE_BF16 = 1 };
/* Precision of the grouped GEMMs: MOE_PREC_NATIVE multiplies in the storage
 * type (bf16, or tf32 for fp32 storage) with fp32 accumulation; MOE_PREC_MXFP8
 * quantises both operands of each grouped GEMM to E4M3 with one E8M0 scale per
 * 32 elements along the reduction axis. */
enum moe_prec { MOE_PREC_NATIVE = 0, MOE_PREC_MXFP8 = 1 };
/* MOE_PREC_MXFP8 needs dtype MOE_BF16 (bf16 storage, outputs and gradients stay bf16).
 * The quantised operands live in the workspace, which is then much larger (about
 * 2*(P + 127*E)*(3d + 3f) + 4*E*d*f bytes). */

typedef struct moe_config {
  int64_t T;     /* tokens */
  int32_t d;     /* model width */
  int32_t E;     /* experts */
  int32_t k;     /* experts per token */
  int32_t f;     /* expert FFN width */
  int32_t dtype; /* enum moe_dtype */
  int32_t prec;  /* enum moe_prec */
} moe_config;

/* (the pages have no counterpart: calling-convention plumbing)
 * Bytes of device workspace every call taking `ws` needs for this config.
 * The workspace holds the error word and small scratch (per-block histograms,
 * a transposed router weight, router-gradient partial sums).  Zero it once
 * (cudaMemset) before its first use; the library keeps it consistent after. */
MOE_API size_t moe_workspace_size(const moe_config *cfg);

/* (the pages have no counterpart: calling-convention plumbing)
 * Bytes of moe_layer_saved.mx_saved for this config: 0 unless prec is MOE_PREC_MXFP8. */
MOE_API size_t moe_mx_saved_bytes(const moe_config *cfg);

/* (the pages have no counterpart: error reporting)
 * Synchronise `stream`, then report and clear the device error word in `ws`.
 * *code receives 0 or an OR of MOE_ERR_DEVICE_* bits. */
MOE_API int moe_get_error(void *ws, moe_stream_t stream, int32_t *code);

/* (the pages have no counterpart: failure detection)
 * Test hook for the kernels' bounded waits.  ns > 0: every grouped GEMM (and the tensor-core
 * router) launched afterwards from this process with single-CTA tiles first waits up to ns
 * nanoseconds on a barrier that nothing arrives on; the wait runs out, every role of the
 * kernel stops, the copies and MMAs already in flight are drained, TMEM is freed, the kernel
 * returns, and MOE_ERR_DEVICE_TIMEOUT is OR-ed into the workspace's error word.  Launches with
 * CTA-pair tiles ignore it.  The outputs of such a launch are undefined.  ns = 0 (the default)
 * turns it off.  ns above MOE_DEBUG_STALL_MAX_NS returns MOE_ERR_INVALID_ARG.  Process-wide,
 * not synchronised with launches already enqueued. */
#define MOE_DEBUG_STALL_MAX_NS 1000000000ull
MOE_API int moe_debug_set_gemm_stall_ns(uint64_t ns);

/* ---------------------------------------------------------------- routing */

/* Router forward (source: qidao123.com, section "新闻原文", 4 of E experts per token; unite.ai, section "Παραλληλισμός, Ακρίβεια και Τεχνικές Μνήμης").
 * logits z = x W_r (+ bias) in fp32; top-k on z, listed by
 * descending logit with equal logits to the lower index; gates
 * g_j = exp(z_j) / sum_j' exp(z_j') over the k selected logits (equal to the
 * full softmax renormalised over the selection).
 *   x [T,d] dtype; w_router [d,E] dtype; bias [E] fp32 or NULL;
 *   logits [T,E] fp32 or NULL (not written); topk_idx [T,k] int32;
 *   topk_gate [T,k] fp32; ws as from moe_workspace_size. */
MOE_API int moe_route_topk(const moe_config *cfg, const void *x, const void *w_router,
                   const float *bias, float *logits, int32_t *topk_idx,
                   float *topk_gate, void *ws, moe_stream_t stream);

/* (source: as moe_route_topk)
 * The router's second half alone: top-k and renormalised gates from given
 * fp32 logits [T,E].  Same selection and gate rule as moe_route_topk. */
MOE_API int moe_topk_gating(const moe_config *cfg, const float *logits, int32_t *topk_idx,
                    float *topk_gate, void *ws, moe_stream_t stream);

/* (source: unite.ai, section "Παραλληλισμός, Ακρίβεια και Τεχνικές Μνήμης" and ettayeb.fr, section "Trois parallélismes, trois optimisations de routage": the routing metadata stays on the GPU so the CPU
 * never waits for a copy back)
 * GPU-resident routing metadata (stable counting sort of the P pairs by expert):
 *   counts[e] = pairs routed to e; offsets[0..E] = exclusive scan of counts
 *   (offsets[E] = P); slot_of_pair[i] = offsets[e] + number of pairs i' < i
 *   with the same expert; pair_of_slot = its inverse.
 *   topk_idx [T,k] int32 in; counts [E], offsets [E+1], slot_of_pair [P],
 *   pair_of_slot [P] int32 out.  Indices outside [0, E) set
 *   MOE_ERR_DEVICE_INDEX and leave the outputs undefined. */
MOE_API int moe_build_offsets(const moe_config *cfg, const int32_t *topk_idx, int32_t *counts,
                      int32_t *offsets, int32_t *slot_of_pair, int32_t *pair_of_slot,
                      void *ws, moe_stream_t stream);

/* moe_build_offsets without a workspace, for callers that cannot allocate device memory
 * (for example a program that gives all GPU memory to its own pool at start-up, or a C
 * caller with no allocator of its own).  Same outputs as moe_build_offsets.
 * (The pages have no counterpart: this is a calling convention, not a step of the method.)
 *   Scratch: a fixed 256 KiB array inside the library, held on every GPU that loads the
 *   library until the process exits; it must hold ceil(T*k/1024) * E int32 histogram
 *   entries (65536 at most), so larger shapes return MOE_ERR_UNSUPPORTED and launch
 *   nothing (e.g. T*k = 262145 at E = 256; T*k = 262144 at E = 256 is the largest fit).
 *   The first call made with a given device current looks up the array's device address
 *   (cudaGetSymbolAddress) and keeps it for that device; make that first call before any
 *   stream capture.  The address kept is the one in the context current at that first call,
 *   which is the device's primary context for callers of the CUDA runtime; a caller that
 *   later makes another context of the same device current (through the driver API) is not
 *   supported.
 *   Every call shares the one array: calls whose work can overlap on the GPU (different
 *   streams, different host threads) race and must be ordered by the caller.
 *   An expert index outside [0, E) leaves the outputs undefined and is not reported.
 *   Allocates nothing (no cudaMalloc, cudaFree or allocating library call). */
MOE_API int moe_build_offsets_noalloc(const moe_config *cfg, const int32_t *topk_idx,
                                      int32_t *counts, int32_t *offsets, int32_t *slot_of_pair,
                                      int32_t *pair_of_slot, moe_stream_t stream);

/* (source: unite.ai, section "Παραλληλισμός, Ακρίβεια και Τεχνικές Μνήμης", and ettayeb.fr,
 * section "Trois parallélismes, trois optimisations de routage": routed rows are written
 * straight into the experts' input buffers, "rowwise" placement)
 * Rowwise dispatch: x_perm[slot_of_pair[t*k+j]] = x[t] (a bit copy).
 *   x [T,d] dtype; slot_of_pair [P]; x_perm [P,d] dtype. */
MOE_API int moe_permute(const moe_config *cfg, const void *x, const int32_t *slot_of_pair,
                void *x_perm, moe_stream_t stream);

/* ------------------------------------------------------ grouped expert FFN */

/* (source: unite.ai, section "Παραλληλισμός, Ακρίβεια και Τεχνικές Μνήμης": one grouped GEMM runs the experts' small matmuls, scheduled from
 * the device)
 * Grouped SwiGLU forward over the expert-contiguous rows of x_perm.  For each
 * expert e and its rows R_e = [offsets[e], offsets[e+1]):
 *   h = x_perm[R_e] Wg[e], u = x_perm[R_e] Wu[e], a = silu(h) * u,
 *   y_perm[R_e] = a Wd[e].
 *   x_perm [P,d]; offsets [E+1]; w_gate, w_up [E,d,f]; w_down [E,f,d];
 *   hu [P,2f] receives h in columns [0,f) and u in [f,2f) (saved for the
 *   backward); a [P,f]; y_perm [P,d].  All dtype; fp32 accumulation.
 * The tile schedule is built on the device from offsets; the host never
 * reads the counts. */
MOE_API int moe_grouped_swiglu_fwd(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                           const void *w_gate, const void *w_up, const void *w_down,
                           void *hu, void *a, void *y_perm, void *ws, moe_stream_t stream);

/* (source: as moe_grouped_swiglu_fwd; the backward is its chain rule)
 * Grouped SwiGLU backward.  Per expert e (rows R_e):
 *   da = dy_perm Wd^T; dh = da * u * silu'(h); du = da * silu(h);
 *   dhu = [dh | du] ([P,2f], written); dx_perm = dh Wg^T + du Wu^T;
 *   dWd[e] = a^T dy_perm; dWg[e] = x_perm^T dh; dWu[e] = x_perm^T du.
 * An expert with no rows gets zero weight gradients.
 *   dy_perm, x_perm [P,d]; hu [P,2f] and a [P,f] from the forward;
 *   dhu [P,2f] out; dx_perm [P,d] out; dw_gate, dw_up [E,d,f] out;
 *   dw_down [E,f,d] out.  All dtype. */
MOE_API int moe_grouped_swiglu_bwd(const moe_config *cfg, const void *dy_perm, const void *x_perm,
                           const void *hu, const void *a, const int32_t *offsets,
                           const void *w_gate, const void *w_up, const void *w_down,
                           void *dhu, void *dx_perm, void *dw_gate, void *dw_up,
                           void *dw_down, void *ws, moe_stream_t stream);

/* MXFP8 quantisation (OCP Microscaling v1.0, as the pages' "MXFP8" is read here):
 * E4M3 codes with one E8M0 scale byte per 32 elements, X = 2^(floor(log2 amax) - 8)
 * clamped to [2^-127, 2^127] (amax = 0 gives 2^-127), v / X rounded to nearest even and
 * saturated to +-448; scale byte = 127 + log2 X.  src is bf16 [rows][cols].
 *   rows variant: blocks of 32 consecutive columns; codes [R'][cols], scales [R'][cols/32].
 *   cols variant: blocks of 32 consecutive rows;    codes [R'][cols], scales [R'/32][cols].
 * offsets == NULL: R' = rows (for the cols variant, a partial last block reads zeros).
 * offsets != NULL ([E+1], as from moe_build_offsets): the rows are E expert groups and are
 *   written into buffers padded to 128 rows per expert; padded row 128*pre[e] + i holds
 *   src row offsets[e] + i for i < count_e and zeros after, pre[e] = sum_{e'<e}
 *   ceil(count_e'/128); the buffers must hold rows_bound >= rows + 127*E rows.
 * cols must be a multiple of 32 (of 128 for the rows variant with offsets).  src and codes
 * 16-byte aligned, scales 4-byte aligned (else MOE_ERR_INVALID_ARG). */
/* FP8 dispatch (unite.ai, "Ai2 κυκλοφορεί το Olmo-Core 3 ...", section "Παραλληλισμός,
 * Ακρίβεια και Τεχνικές Μνήμης": MXFP8 also for the data moved between experts): the
 * permute of moe_permute (x_perm [P,d] bf16, a bit copy of each routed row) and, in the same
 * pass, each routed row in MXFP8 with blocks of 32 along d, written as moe_mx_quantize_rows
 * with offsets writes it: codes [rows_bound][d] and scales [rows_bound][d/32], padded row
 * 128*pre[e] + (slot - offsets[e]).  Rows of the padding past an expert's count are left
 * as they were.  bf16 only (else MOE_ERR_UNSUPPORTED); rows_bound >= T*k + 127*E; x, x_perm,
 * codes 16-byte aligned, slot_of_pair, offsets, scales 4-byte aligned.  offsets from
 * moe_build_offsets. */
MOE_API int moe_permute_mxfp8(const moe_config *cfg, const void *x, const int32_t *slot_of_pair,
                              const int32_t *offsets, void *x_perm, int64_t rows_bound,
                              uint8_t *codes, uint8_t *scales, moe_stream_t stream);

/* FP8 dispatch in both orientations (same passage): each routed row of x is read once, in
 * slot order through pair_of_slot, and written in MXFP8 twice on the expert-padded layout
 * (padded row 128*pre[e] + i holds x[pair_of_slot[offsets[e] + i] / k] for i < count_e and
 * zeros after, up to 128*pre[E]):
 *   codes_r [rows_bound][d], scales_r [rows_bound][d/32]: blocks of 32 along d (the forward
 *     GEMM's operand), as moe_mx_quantize_rows with offsets;
 *   codes_c [rows_bound][d], scales_c [rows_bound/32][d]: blocks of 32 padded rows (the
 *     weight gradient's operand), as moe_mx_quantize_cols with offsets.
 * x_perm [P,d] or NULL: the bf16 bit copy of moe_permute as well.  The pad rows are written
 * (zeros, scale byte 0); rows past 128*pre[E] are left as they were.  bf16 only (else
 * MOE_ERR_UNSUPPORTED); rows_bound >= T*k + 127*E (else MOE_ERR_INVALID_ARG); x, x_perm, codes 16-byte aligned, pair_of_slot, offsets, scales
 * 4-byte aligned; pair_of_slot and offsets from moe_build_offsets. */
MOE_API int moe_dispatch_mxfp8(const moe_config *cfg, const void *x, const int32_t *pair_of_slot,
                               const int32_t *offsets, int64_t rows_bound, void *x_perm,
                               uint8_t *codes_r, uint8_t *scales_r, uint8_t *codes_c,
                               uint8_t *scales_c, moe_stream_t stream);

MOE_API int moe_mx_quantize_rows(const void *src, int64_t rows, int32_t cols, const int32_t *offsets,
                                 int32_t E, int64_t rows_bound, uint8_t *codes, uint8_t *scales,
                                 moe_stream_t stream);
MOE_API int moe_mx_quantize_cols(const void *src, int64_t rows, int32_t cols, const int32_t *offsets,
                                 int32_t E, int64_t rows_bound, uint8_t *codes, uint8_t *scales,
                                 moe_stream_t stream);

/* ---------------------------------------------------------------- combine */

/* (source: unite.ai, section "Παραλληλισμός, Ακρίβεια και Τεχνικές Μνήμης": the inverse of the rowwise placement, weighted by the gates)
 * Gate-weighted unpermute: y[t] = sum_j topk_gate[t,j] * y_perm[slot_of_pair[t*k+j]],
 * accumulated in fp32.  y_perm [P,d]; y [T,d] dtype. */
MOE_API int moe_unpermute_combine(const moe_config *cfg, const void *y_perm,
                          const int32_t *slot_of_pair, const float *topk_gate, void *y,
                          moe_stream_t stream);

/* (source: as moe_unpermute_combine; its chain rule)
 * Backward of the combine: dy_perm[slot(t,j)] = g[t,j] * dy[t];
 * dgate[t,j] = <dy[t], y_perm[slot(t,j)]> (fp32).
 *   dy [T,d]; y_perm [P,d]; dy_perm [P,d] out; dgate [T,k] fp32 out. */
MOE_API int moe_combine_bwd(const moe_config *cfg, const void *dy, const void *y_perm,
                    const int32_t *slot_of_pair, const float *topk_gate, void *dy_perm,
                    float *dgate, moe_stream_t stream);

/* The combine's backward with its output dispatched in MXFP8 (unite.ai, section
 * "Παραλληλισμός, Ακρίβεια και Τεχνικές Μνήμης": MXFP8 for the data moved between experts):
 * for each slot, in the order of pair_of_slot, dy_perm row = bf16(g * dy[t]) (the fp32
 * product rounded to bf16) and dgate[t,j] = <dy[t], y_perm[slot]> (fp32); the bf16 row is
 * then written in MXFP8 in both orientations exactly as moe_dispatch_mxfp8 writes x's rows
 * (codes_r/scales_r along d, codes_c/scales_c down the padded token axis).  dy_perm [P,d] or
 * NULL: the bf16 rows as well.  Arguments, alignment and errors as moe_dispatch_mxfp8, with
 * y_perm [P,d] bf16, topk_gate [T,k] fp32 and dgate [T,k] fp32 out (4-byte aligned). */
MOE_API int moe_combine_bwd_mxfp8(const moe_config *cfg, const void *dy, const void *y_perm,
                                  const int32_t *pair_of_slot, const int32_t *offsets,
                                  const float *topk_gate, int64_t rows_bound, void *dy_perm,
                                  float *dgate, uint8_t *codes_r, uint8_t *scales_r,
                                  uint8_t *codes_c, uint8_t *scales_c, moe_stream_t stream);

/* (source: as moe_permute; its chain rule)
 * Backward of the permute: dx[t] = sum_j dx_perm[slot(t,j)] (fp32 sum).
 *   dx_perm [P,d]; dx [T,d] out. */
MOE_API int moe_unpermute_sum(const moe_config *cfg, const void *dx_perm,
                      const int32_t *slot_of_pair, void *dx, moe_stream_t stream);

/* (source: as moe_route_topk; its chain rule)
 * Router backward.  dz[t,S_j] = g_j (dgate_j - sum_j' g_j' dgate_j'), zero on
 * unselected experts; dw_router = x^T dz ([d,E] fp32, overwritten);
 * dx[t] += dz[t] W_r^T (dx [T,d] dtype, read and written). */
MOE_API int moe_route_bwd(const moe_config *cfg, const float *dgate, const float *topk_gate,
                  const int32_t *topk_idx, const void *x, const void *w_router, void *dx,
                  float *dw_router, void *ws, moe_stream_t stream);

/* ------------------------------------------------------------ whole layer */

typedef struct moe_layer_weights {
  const void *w_router; /* [d,E] dtype */
  const float *bias;    /* [E] fp32 additive logit bias, or NULL */
  const void *w_gate;   /* [E,d,f] */
  const void *w_up;     /* [E,d,f] */
  const void *w_down;   /* [E,f,d] */
  /* Optional shared expert (bigchange.ai, "Olmo-core 3 открывает стек обучения MoE от
   * Ai2 ...", section "Что инженер может попробовать на практике": the published production
   * rows route each token to four experts and also use one shared expert).  A SwiGLU of
   * the routed experts' shape that every token passes through; its output is added to the
   * gate-weighted sum of the routed experts with weight 1.  All three NULL: none. */
  const void *w_shared_gate; /* [d,f] */
  const void *w_shared_up;   /* [d,f] */
  const void *w_shared_down; /* [f,d] */
} moe_layer_weights;

/* Buffers the forward fills and the backward reads (caller-owned). */
typedef struct moe_layer_saved {
  float *logits;          /* [T,E] fp32, or NULL */
  int32_t *topk_idx;      /* [T,k] */
  float *topk_gate;       /* [T,k] */
  int32_t *counts;        /* [E] */
  int32_t *offsets;       /* [E+1] */
  int32_t *slot_of_pair;  /* [P] */
  int32_t *pair_of_slot;  /* [P] */
  void *x_perm;           /* [P,d]; unused (may be NULL) with mx_saved */
  void *hu;               /* [P,2f] (h | u), or NULL: the backward recomputes them */
  void *a;                /* [P,f] */
  void *y_perm;           /* [P,d] */
  void *shared_hu;        /* [T,2f] with a shared expert, or NULL: recomputed */
  void *shared_a;         /* [T,f] with a shared expert */
  /* MOE_PREC_MXFP8 only, or NULL: moe_mx_saved_bytes(cfg) bytes (256-byte aligned) that the
   * forward fills with MXFP8 copies (E4M3 codes with E8M0 scales, the layout is internal) the
   * backward reads instead of quantising again: the routed experts' weights in the orientation
   * of every GEMM that reads them, the routed rows of x along d and along the token axis, and
   * a along the token axis.  The routed rows then move in MXFP8 only (the FP8 dispatch): x_perm
   * is neither written nor read, and the router's weight gradient reads x through
   * pair_of_slot.  The weights must not change between the two calls.  NULL: the forward also
   * writes the bf16 x_perm, and each call quantises what it needs in the workspace. */
  void *mx_saved;
} moe_layer_saved;

/* Outputs of the backward, plus its intermediates (caller-owned). */
typedef struct moe_layer_grads {
  void *dx;          /* [T,d] */
  float *dw_router;  /* [d,E] fp32, or NULL to skip the router backward */
  void *dw_gate;     /* [E,d,f] */
  void *dw_up;       /* [E,d,f] */
  void *dw_down;     /* [E,f,d] */
  void *dy_perm;     /* [P,d] intermediate; unused (may be NULL) with MOE_PREC_MXFP8, where the
                        combine's backward writes it in MXFP8 only */
  float *dgate;      /* [T,k] intermediate */
  void *dhu;         /* [P,2f] intermediate (also holds recomputed h | u); with MOE_PREC_MXFP8
                        [dh | du] is kept in MXFP8 only and dhu holds no defined values after
                        the call (it is still required: the recompute's scratch) */
  void *dx_perm;     /* [P,d] intermediate */
  void *dw_shared_gate; /* [d,f] with a shared expert */
  void *dw_shared_up;   /* [d,f] */
  void *dw_shared_down; /* [f,d] */
  void *shared_dhu;     /* [T,2f] intermediate with a shared expert */
} moe_layer_grads;

/* Whole forward: route_topk -> build_offsets -> permute -> grouped SwiGLU ->
 * unpermute_combine, all enqueued on `stream` with no host synchronisation.
 *   x [T,d]; y [T,d] out.
 * With a shared expert, its SwiGLU runs through the grouped GEMM as one group of all T
 * tokens (x itself is that group's buffer), writes y, and the combine adds the routed
 * experts' gate-weighted rows to it.
 * Recompute (bigchange.ai, section "Три числа, три знаменателя": the largest published
 * row recomputes activations in every layer): saved->hu == NULL keeps only a; the
 * backward then recomputes h | u from x_perm (one extra grouped GEMM) into g->dhu and
 * runs the SwiGLU backward in place there.  The same holds for saved->shared_hu. */
MOE_API int moe_layer_fwd(const moe_config *cfg, const moe_layer_weights *w, const void *x, void *y,
                  const moe_layer_saved *saved, void *ws, moe_stream_t stream);

/* Forward from given routing (e.g. uniform random routing with gates 1/k):
 * skips the router; saved->topk_idx and saved->topk_gate are inputs. */
MOE_API int moe_layer_fwd_routed(const moe_config *cfg, const moe_layer_weights *w, const void *x,
                         void *y, const moe_layer_saved *saved, void *ws, moe_stream_t stream);

/* Whole backward from dy [T,d]: combine_bwd -> grouped SwiGLU backward ->
 * unpermute_sum (+ router backward when g->dw_router is not NULL). */
MOE_API int moe_layer_bwd(const moe_config *cfg, const moe_layer_weights *w, const void *x,
                  const void *dy, const moe_layer_saved *saved, const moe_layer_grads *g,
                  void *ws, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
