// Router (logits, softmax top-k, renormalised gates) and GPU-resident routing
// metadata (counts, exclusive-scan offsets, stable slot maps).
//
// Method: unite.ai "Ai2 κυκλοφορεί το Olmo-Core 3 ...", section "Παραλληλισμός,
// Ακρίβεια και Τεχνικές Μνήμης": routing metadata stays on the GPU so the CPU
// never waits for a copy back; ettayeb.fr "Olmo-core 3 ouvre l'entraînement des
// MoE ...", section "Trois parallélismes, trois optimisations de routage".
// qidao123.com "Ai2开源Olmo-core 3 ...", section "新闻原文": 4 of E experts per token.
#include "common.cuh"

namespace moe {

// ------------------------------------------------------------------------------------
// Warp-level top-k over one token's logits held across the lanes.
// Lane l holds experts l + 32*j, j < EPT.  Order: larger logit first, equal logits to
// the lower index.  NaN never beats a number (it is only picked when nothing else is
// left), so the k indices are always distinct and in range.
// ------------------------------------------------------------------------------------
struct Cand {
  float v;
  int i;  // expert index, or INT_MAX when the lane has nothing left
};

// A strict total order on candidates: numbers before NaNs, larger first, then lower index.
__device__ __forceinline__ bool better(const Cand &a, const Cand &b) {
  if (a.i == INT_MAX) return false;
  if (b.i == INT_MAX) return true;
  const bool an = a.v != a.v, bn = b.v != b.v;
  if (an != bn) return bn;
  if (an) return a.i < b.i;
  return a.v > b.v || (a.v == b.v && a.i < b.i);
}

template <int EPT>
__device__ __forceinline__ void warp_topk_write(const float (&v)[EPT], int E, int k, int64_t t,
                                                int32_t *idx_out, float *gate_out, int *err) {
  const int lane = threadIdx.x & 31;
  unsigned taken = 0;
  float sel_v[MAX_K];
  int sel_i[MAX_K];
  bool nan_seen = false;
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    int e = lane + 32 * j;
    if (e < E && v[j] != v[j]) nan_seen = true;
  }
#pragma unroll
  for (int r = 0; r < MAX_K; ++r) {
    if (r < k) {
      Cand best{0.f, INT_MAX};
#pragma unroll
      for (int j = 0; j < EPT; ++j) {
        int e = lane + 32 * j;
        Cand c{v[j], (e < E && !((taken >> j) & 1u)) ? e : INT_MAX};
        if (better(c, best)) best = c;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        Cand other{__shfl_xor_sync(0xffffffffu, best.v, o), __shfl_xor_sync(0xffffffffu, best.i, o)};
        if (better(other, best)) best = other;
      }
      sel_v[r] = best.v;
      sel_i[r] = best.i;
      if ((best.i & 31) == lane) taken |= 1u << (best.i >> 5);
    }
  }
  if (__any_sync(0xffffffffu, nan_seen) && lane == 0) set_error(err, MOE_ERR_DEVICE_NAN);
  // gates: softmax over the selected logits (largest first, so sel_v[0] is the max)
  float m = sel_v[0];
  float s = 0.f;
  float ex[MAX_K];
#pragma unroll
  for (int r = 0; r < MAX_K; ++r) {
    if (r < k) { ex[r] = expf(sel_v[r] - m); s += ex[r]; }
  }
  float inv = 1.0f / s;
#pragma unroll
  for (int r = 0; r < MAX_K; ++r) {
    if (r < k && lane == r) {
      idx_out[t * k + r] = sel_i[r];
      gate_out[t * k + r] = ex[r] * inv;
    }
  }
}

// ------------------------------------------------------------------------------------
// Router: z = x W_r (+ b) on CUDA cores in fp32, then top-k per token.
// CTA = 256 threads = 8 warps, 32 tokens.  Warp w owns tokens 4w..4w+3; lane l owns
// experts [l*EPT, l*EPT+EPT).  The d axis is walked in chunks of KC through shared
// memory (x chunk transposed to [KC][32], W_r chunk as [KC][32*EPT]).
// ------------------------------------------------------------------------------------
constexpr int RT_TOK = 32;
constexpr int RT_KC = 32;

template <typename T, int EPT>
__global__ void __launch_bounds__(256) route_topk_kernel(const T *__restrict__ x,
                                                         const T *__restrict__ w_r,
                                                         const float *__restrict__ bias,
                                                         float *__restrict__ logits,
                                                         int32_t *__restrict__ idx,
                                                         float *__restrict__ gate, int64_t T_,
                                                         int d, int E, int k, int *err) {
  constexpr int EP = 32 * EPT;
  constexpr int XS_LD = RT_TOK + 4;  // row pitch keeps float4 alignment, spreads banks
  constexpr int WZ = (RT_KC * EP > RT_TOK * (EP + 1)) ? RT_KC * EP : RT_TOK * (EP + 1);
  __shared__ __align__(16) float xs[RT_KC * XS_LD];
  __shared__ __align__(16) float wz[WZ];  // W_r chunk [KC][EP] during the GEMM, logits [32][EP+1] after
  float *ws = wz;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t t0 = (int64_t)blockIdx.x * RT_TOK;

  float acc[4][EPT];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < EPT; ++b) acc[a][b] = 0.f;

  for (int k0 = 0; k0 < d; k0 += RT_KC) {
    // x chunk: 32 tokens x 32 columns, stored transposed
    for (int i = tid; i < RT_TOK * RT_KC; i += 256) {
      int tt = i / RT_KC, kk = i % RT_KC;
      int64_t t = t0 + tt;
      xs[kk * XS_LD + tt] = (t < T_) ? to_f(x[t * d + k0 + kk]) : 0.f;
    }
    for (int i = tid; i < RT_KC * EP; i += 256) {
      int kk = i / EP, e = i % EP;
      ws[kk * EP + e] = (e < E) ? to_f(w_r[(int64_t)(k0 + kk) * E + e]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < RT_KC; ++kk) {
      float4 xv = *reinterpret_cast<const float4 *>(&xs[kk * XS_LD + warp * 4]);
      float wv[EPT];
      if constexpr (EPT % 4 == 0) {
#pragma unroll
        for (int b = 0; b < EPT; b += 4) {
          float4 q = *reinterpret_cast<const float4 *>(&ws[kk * EP + lane * EPT + b]);
          wv[b] = q.x; wv[b + 1] = q.y; wv[b + 2] = q.z; wv[b + 3] = q.w;
        }
      } else {
#pragma unroll
        for (int b = 0; b < EPT; ++b) wv[b] = ws[kk * EP + lane * EPT + b];
      }
#pragma unroll
      for (int b = 0; b < EPT; ++b) {
        acc[0][b] = fmaf(xv.x, wv[b], acc[0][b]);
        acc[1][b] = fmaf(xv.y, wv[b], acc[1][b]);
        acc[2][b] = fmaf(xv.z, wv[b], acc[2][b]);
        acc[3][b] = fmaf(xv.w, wv[b], acc[3][b]);
      }
    }
    __syncthreads();
  }
  // (the loop above ends with a barrier, so the W_r chunk buffer can now hold logits)
  float *zs = wz;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    int tt = warp * 4 + a;
    int64_t t = t0 + tt;
#pragma unroll
    for (int b = 0; b < EPT; ++b) {
      int e = lane * EPT + b;
      float z = acc[a][b];
      if (e < E) {
        if (bias) z += bias[e];
        if (logits && t < T_) logits[t * E + e] = z;
      }
      zs[tt * (EP + 1) + e] = z;
    }
  }
  __syncthreads();
  // top-k: warp w handles its own 4 tokens; lane l now holds experts l + 32*j
#pragma unroll 1
  for (int a = 0; a < 4; ++a) {
    int tt = warp * 4 + a;
    int64_t t = t0 + tt;
    if (t >= T_) break;
    float v[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) v[j] = zs[tt * (EP + 1) + lane + 32 * j];
    warp_topk_write<EPT>(v, E, k, t, idx, gate, err);
  }
}

// Top-k from given logits: one warp per token.
template <int EPT>
__global__ void __launch_bounds__(256) topk_gating_kernel(const float *__restrict__ logits,
                                                          int32_t *__restrict__ idx,
                                                          float *__restrict__ gate, int64_t T_,
                                                          int E, int k, int *err) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T_) return;
  float v[EPT];
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    int e = lane + 32 * j;
    v[j] = (e < E) ? logits[t * E + e] : 0.f;
  }
  warp_topk_write<EPT>(v, E, k, t, idx, gate, err);
}

static int ept_of(int E) {
  int ep = (E + 31) / 32;
  return ep <= 1 ? 1 : ep <= 2 ? 2 : ep <= 4 ? 4 : 8;
}

template <typename T>
static cudaError_t route_dispatch(const Shape &s, const void *x, const void *w_r, const float *bias,
                                  float *logits, int32_t *idx, float *gate, int *err,
                                  cudaStream_t st) {
  dim3 grid((unsigned)((s.T + RT_TOK - 1) / RT_TOK));
  const T *xp = static_cast<const T *>(x);
  const T *wp = static_cast<const T *>(w_r);
  switch (ept_of(s.E)) {
    case 1: route_topk_kernel<T, 1><<<grid, 256, 0, st>>>(xp, wp, bias, logits, idx, gate, s.T, s.d, s.E, s.k, err); break;
    case 2: route_topk_kernel<T, 2><<<grid, 256, 0, st>>>(xp, wp, bias, logits, idx, gate, s.T, s.d, s.E, s.k, err); break;
    case 4: route_topk_kernel<T, 4><<<grid, 256, 0, st>>>(xp, wp, bias, logits, idx, gate, s.T, s.d, s.E, s.k, err); break;
    default: route_topk_kernel<T, 8><<<grid, 256, 0, st>>>(xp, wp, bias, logits, idx, gate, s.T, s.d, s.E, s.k, err); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_route_topk(const Shape &s, const void *x, const void *w_r, const float *bias,
                              float *logits, int32_t *idx, float *gate, int *err, cudaStream_t st) {
  if (s.T == 0) return cudaSuccess;
  if (s.dtype == MOE_BF16 && s.E % 8 == 0) {
    // the tensor-core router; its host-side failures come back as a CUDA error
    return launch_router_tc(s, x, w_r, bias, logits, idx, gate, err, st) == MOE_OK ? cudaSuccess
                                                                                   : cudaErrorLaunchFailure;
  }
  if (s.dtype == MOE_BF16) return route_dispatch<bf16>(s, x, w_r, bias, logits, idx, gate, err, st);
  return route_dispatch<float>(s, x, w_r, bias, logits, idx, gate, err, st);
}

cudaError_t launch_topk_gating(const Shape &s, const float *logits, int32_t *idx, float *gate,
                               int *err, cudaStream_t st) {
  if (s.T == 0) return cudaSuccess;
  dim3 grid((unsigned)((s.T + 7) / 8));
  switch (ept_of(s.E)) {
    case 1: topk_gating_kernel<1><<<grid, 256, 0, st>>>(logits, idx, gate, s.T, s.E, s.k, err); break;
    case 2: topk_gating_kernel<2><<<grid, 256, 0, st>>>(logits, idx, gate, s.T, s.E, s.k, err); break;
    case 4: topk_gating_kernel<4><<<grid, 256, 0, st>>>(logits, idx, gate, s.T, s.E, s.k, err); break;
    default: topk_gating_kernel<8><<<grid, 256, 0, st>>>(logits, idx, gate, s.T, s.E, s.k, err); break;
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------
// Routing metadata: a stable counting sort of the P routed pairs by expert, in three
// launches with no host synchronisation:
//   1. per-block histograms over chunks of SCATTER_CHUNK pairs;
//   2. one block: counts, exclusive-scan offsets, and each (block, expert) base slot;
//   3. per block, the stable rank of every pair among its expert's pairs
//      (warp-sliced histograms, then __match_any_sync + popc inside each warp).
// ------------------------------------------------------------------------------------
constexpr int SC_THREADS = 256;
constexpr int SC_WARPS = SC_THREADS / 32;
constexpr int SC_PER_WARP = SCATTER_CHUNK / SC_WARPS;  // 128 pairs, 4 rounds of 32

__global__ void __launch_bounds__(SC_THREADS) offsets_hist_kernel(const int32_t *__restrict__ idx,
                                                                  int64_t P, int E,
                                                                  int32_t *__restrict__ block_counts,
                                                                  int *err) {
  __shared__ int hist[MAX_E];
  for (int e = threadIdx.x; e < E; e += SC_THREADS) hist[e] = 0;
  __syncthreads();
  int64_t base = (int64_t)blockIdx.x * SCATTER_CHUNK;
  for (int i = threadIdx.x; i < SCATTER_CHUNK; i += SC_THREADS) {
    int64_t p = base + i;
    if (p < P) {
      int e = idx[p];
      if ((unsigned)e < (unsigned)E) atomicAdd(&hist[e], 1);
      else set_error(err, MOE_ERR_DEVICE_INDEX);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += SC_THREADS)
    block_counts[(int64_t)blockIdx.x * E + e] = hist[e];
}

// One block of 256 threads; thread e < E walks its column of block_counts.
__global__ void __launch_bounds__(256) offsets_scan_kernel(int32_t *__restrict__ block_counts,
                                                           int nblocks, int E, int64_t P,
                                                           int32_t *__restrict__ counts,
                                                           int32_t *__restrict__ offsets) {
  __shared__ int warp_tot[8];
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  int c = 0;
  if (e < E)
    for (int b = 0; b < nblocks; ++b) c += block_counts[(int64_t)b * E + e];
  // block-wide exclusive scan of c over e
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += warp_tot[w];
  int excl = wbase + incl - c;
  if (e < E) {
    counts[e] = c;
    offsets[e] = excl;
    if (e == E - 1) offsets[E] = (int32_t)P;
    int run = excl;
    for (int b = 0; b < nblocks; ++b) {
      int32_t *p = &block_counts[(int64_t)b * E + e];
      int v = *p;
      *p = run;  // becomes this block's first slot for expert e
      run += v;
    }
  }
}

__global__ void __launch_bounds__(SC_THREADS) offsets_scatter_kernel(
    const int32_t *__restrict__ idx, int64_t P, int E, const int32_t *__restrict__ block_base,
    int32_t *__restrict__ slot_of_pair, int32_t *__restrict__ pair_of_slot) {
  __shared__ int wh[SC_WARPS][MAX_E];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < SC_WARPS * MAX_E; i += SC_THREADS) (&wh[0][0])[i] = 0;
  __syncthreads();
  const int64_t wbase = (int64_t)blockIdx.x * SCATTER_CHUNK + (int64_t)warp * SC_PER_WARP;
  const unsigned lt_mask = (1u << lane) - 1u;
  // pass 1: this warp's per-expert counts
#pragma unroll 1
  for (int r = 0; r < SC_PER_WARP; r += 32) {
    int64_t p = wbase + r + lane;
    int e = (p < P) ? idx[p] : -1;
    if ((unsigned)e >= (unsigned)E) e = -1;
    unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (peers & lt_mask) == 0) wh[warp][e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // exclusive prefix over the warps of this block, on top of the block's base slots
  for (int e = threadIdx.x; e < E; e += SC_THREADS) {
    int run = block_base[(int64_t)blockIdx.x * E + e];
    for (int w = 0; w < SC_WARPS; ++w) {
      int v = wh[w][e];
      wh[w][e] = run;
      run += v;
    }
  }
  __syncthreads();
  // pass 2: stable ranks in pair order
#pragma unroll 1
  for (int r = 0; r < SC_PER_WARP; r += 32) {
    int64_t p = wbase + r + lane;
    int e = (p < P) ? idx[p] : -1;
    if ((unsigned)e >= (unsigned)E) e = -1;
    unsigned peers = __match_any_sync(0xffffffffu, e);
    int slot = 0;
    if (e >= 0) slot = wh[warp][e] + __popc(peers & lt_mask);
    __syncwarp();
    if (e >= 0) {
      slot_of_pair[p] = slot;
      pair_of_slot[slot] = (int32_t)p;
      if ((peers & lt_mask) == 0) wh[warp][e] += __popc(peers);
    }
    __syncwarp();
  }
}

cudaError_t launch_build_offsets(const Shape &s, const int32_t *idx, int32_t *counts,
                                 int32_t *offsets, int32_t *slot_of_pair, int32_t *pair_of_slot,
                                 int32_t *block_counts, int *err, cudaStream_t st) {
  int64_t P = s.P();
  int nb = (int)((P + SCATTER_CHUNK - 1) / SCATTER_CHUNK);
  if (nb > 0) {
    offsets_hist_kernel<<<nb, SC_THREADS, 0, st>>>(idx, P, s.E, block_counts, err);
  }
  offsets_scan_kernel<<<1, 256, 0, st>>>(block_counts, nb, s.E, P, counts, offsets);
  if (nb > 0) {
    offsets_scatter_kernel<<<nb, SC_THREADS, 0, st>>>(idx, P, s.E, block_counts, slot_of_pair,
                                                      pair_of_slot);
  }
  return cudaGetLastError();
}

}  // namespace moe
