// Row-wise, HBM-bound steps of the layer: rowwise dispatch (permute), gate-weighted
// unpermute-combine, their backwards, and the router backward.
//
// Method: unite.ai "Ai2 κυκλοφορεί το Olmo-Core 3 ...", section "Παραλληλισμός,
// Ακρίβεια και Τεχνικές Μνήμης" and ettayeb.fr "Olmo-core 3 ouvre l'entraînement des
// MoE ...", section "Trois parallélismes, trois optimisations de routage": routed rows
// are placed straight into each expert's contiguous input buffer.  The combine is the
// inverse step, weighting each of a token's k expert outputs by its gate.
//
// Every kernel gives one warp to one token and moves its rows as 16-byte vectors
// (8 bf16 or 4 fp32 per lane per access), so each row access is fully coalesced.
#include <algorithm>
#include <atomic>

#include "common.cuh"

namespace moe {

constexpr int ROW_THREADS = 256;
constexpr int ROW_WARPS = ROW_THREADS / 32;

// Broadcast the k slots (and optionally gates) of token t to every lane.
__device__ __forceinline__ int64_t lane_slot(const int32_t *sop, int64_t t, int k) {
  int lane = threadIdx.x & 31;
  return lane < k ? (int64_t)sop[t * k + lane] : 0;
}

// x_perm[slot(t,j)] = x[t]
__global__ void __launch_bounds__(ROW_THREADS) permute_kernel(const uint4 *__restrict__ x,
                                                              const int32_t *__restrict__ sop,
                                                              uint4 *__restrict__ x_perm,
                                                              int64_t T, int k, int nv) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * ROW_WARPS + (threadIdx.x >> 5);
  if (t >= T) return;
  int64_t my_slot = lane_slot(sop, t, k);
  int64_t slot[MAX_K];
#pragma unroll
  for (int j = 0; j < MAX_K; ++j) slot[j] = __shfl_sync(0xffffffffu, my_slot, j);
  const uint4 *src = x + t * nv;
  for (int v0 = 0; v0 < nv; v0 += 32 * 4) {
    uint4 buf[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      int v = v0 + u * 32 + lane;
      if (v < nv) buf[u] = __ldg(src + v);
    }
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) {
      if (j < k) {
        uint4 *dst = x_perm + slot[j] * nv;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          int v = v0 + u * 32 + lane;
          if (v < nv) dst[v] = buf[u];
        }
      }
    }
  }
}

// y[t] = sum_j g[t,j] * y_perm[slot(t,j)]   (fp32 accumulation).  KC >= k: all k rows'
// vectors of a pass are loaded before the first is used, so k loads are in flight at once.
template <typename T, int KC>
__global__ void __launch_bounds__(ROW_THREADS) combine_kernel(const uint4 *__restrict__ y_perm,
                                                              const int32_t *__restrict__ sop,
                                                              const float *__restrict__ gate,
                                                              uint4 *__restrict__ y, int64_t Tn,
                                                              int k, int nv, bool accumulate) {
  constexpr int N = Vec<T>::N;
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * ROW_WARPS + (threadIdx.x >> 5);
  if (t >= Tn) return;
  const int my_slot = lane < k ? sop[t * k + lane] : 0;
  const float my_g = lane < k ? gate[t * k + lane] : 0.f;
  int slot[KC];
  float g[KC];
#pragma unroll
  for (int j = 0; j < KC; ++j) {
    slot[j] = __shfl_sync(0xffffffffu, my_slot, j);
    g[j] = __shfl_sync(0xffffffffu, my_g, j);
  }
  for (int v0 = 0; v0 < nv; v0 += 64) {
    float acc[2][N];
    uint4 raw[2][KC];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int v = v0 + u * 32 + lane;
      if (accumulate && v < nv) {
        Vec<T>::load(y[t * nv + v], acc[u]);   // y already holds the shared expert's output
      } else {
#pragma unroll
        for (int i = 0; i < N; ++i) acc[u][i] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < KC; ++j)
        raw[u][j] = (j < k && v < nv) ? __ldg(y_perm + (int64_t)slot[j] * nv + v) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v >= nv) continue;
#pragma unroll
      for (int j = 0; j < KC; ++j) {
        if (j < k) {
          float f[N];
          Vec<T>::load(raw[u][j], f);
#pragma unroll
          for (int i = 0; i < N; ++i) acc[u][i] = fmaf(g[j], f[i], acc[u][i]);
        }
      }
      y[t * nv + v] = Vec<T>::store(acc[u]);
    }
  }
}

// dy_perm[slot(t,j)] = g[t,j] dy[t];  dgate[t,j] = <dy[t], y_perm[slot(t,j)]>
template <typename T>
__global__ void __launch_bounds__(ROW_THREADS) combine_bwd_kernel(
    const uint4 *__restrict__ dy, const uint4 *__restrict__ y_perm, const int32_t *__restrict__ sop,
    const float *__restrict__ gate, uint4 *__restrict__ dy_perm, float *__restrict__ dgate,
    int64_t Tn, int k, int nv) {
  constexpr int N = Vec<T>::N;
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * ROW_WARPS + (threadIdx.x >> 5);
  if (t >= Tn) return;
  int64_t my_slot = lane_slot(sop, t, k);
  float my_g = lane < k ? gate[t * k + lane] : 0.f;
  int64_t slot[MAX_K];
  float g[MAX_K], dot[MAX_K];
#pragma unroll
  for (int j = 0; j < MAX_K; ++j) {
    slot[j] = __shfl_sync(0xffffffffu, my_slot, j);
    g[j] = __shfl_sync(0xffffffffu, my_g, j);
    dot[j] = 0.f;
  }
  // two 16-byte vectors per lane per pass, so that more loads are in flight
  for (int v0 = 0; v0 < nv; v0 += 64) {
    float fd[2][N];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v < nv) Vec<T>::load(__ldg(dy + t * nv + v), fd[u]);
    }
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) {
      if (j < k) {
        uint4 ry[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int v = v0 + u * 32 + lane;
          if (v < nv) ry[u] = __ldg(y_perm + slot[j] * nv + v);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int v = v0 + u * 32 + lane;
          if (v < nv) {
            float fy[N], o[N];
            Vec<T>::load(ry[u], fy);
#pragma unroll
            for (int i = 0; i < N; ++i) {
              dot[j] = fmaf(fd[u][i], fy[i], dot[j]);
              o[i] = g[j] * fd[u][i];
            }
            dy_perm[slot[j] * nv + v] = Vec<T>::store(o);
          }
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < MAX_K; ++j) {
    if (j < k) {
      float s = dot[j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) dgate[t * k + j] = s;
    }
  }
}

// dz_j = g_j (dg_j - sum_j' g_j' dg_j') for token t, computed by every lane.
__device__ __forceinline__ void token_dz(const float *dgate, const float *gate, int64_t t, int k,
                                         float (&dz)[MAX_K]) {
  float inner = 0.f;
#pragma unroll
  for (int j = 0; j < MAX_K; ++j)
    if (j < k) inner = fmaf(gate[t * k + j], dgate[t * k + j], inner);
#pragma unroll
  for (int j = 0; j < MAX_K; ++j)
    dz[j] = (j < k) ? gate[t * k + j] * (dgate[t * k + j] - inner) : 0.f;
}

// dx[t] = [dx[t]] + sum_j dx_perm[slot(t,j)] + sum_j dz_j W_r^T[e_j]
// (dx_perm / w_rt may each be null; accumulate reads the old dx).  w_rt is the transposed
// router weight [E][d] in the storage type T (an exact copy of W_r's values).
template <typename T>
__global__ void __launch_bounds__(ROW_THREADS) unpermute_sum_kernel(
    const uint4 *__restrict__ dx_perm, const int32_t *__restrict__ sop,
    const float *__restrict__ dgate, const float *__restrict__ gate, const int32_t *__restrict__ idx,
    const uint4 *__restrict__ w_rt, bool accumulate, uint4 *__restrict__ dx, int64_t Tn, int k,
    int nv) {
  constexpr int N = Vec<T>::N;
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * ROW_WARPS + (threadIdx.x >> 5);
  if (t >= Tn) return;
  int64_t slot[MAX_K];
  int e[MAX_K];
  float dz[MAX_K];
  if (dx_perm) {
    int64_t my_slot = lane_slot(sop, t, k);
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) slot[j] = __shfl_sync(0xffffffffu, my_slot, j);
  }
  if (w_rt) {
    token_dz(dgate, gate, t, k, dz);
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) e[j] = (j < k) ? idx[t * k + j] : 0;
  }
  for (int v = lane; v < nv; v += 32) {
    float acc[N];
    if (accumulate) {
      Vec<T>::load(dx[t * nv + v], acc);
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) acc[i] = 0.f;
    }
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) {
      if (j < k) {
        float f[N];
        if (dx_perm) {
          Vec<T>::load(__ldg(dx_perm + slot[j] * nv + v), f);
#pragma unroll
          for (int i = 0; i < N; ++i) acc[i] += f[i];
        }
        if (w_rt) {
          Vec<T>::load(__ldg(w_rt + (int64_t)e[j] * nv + v), f);
#pragma unroll
          for (int i = 0; i < N; ++i) acc[i] = fmaf(dz[j], f[i], acc[i]);
        }
      }
    }
    dx[t * nv + v] = Vec<T>::store(acc);
  }
}

// The same sum with the router term, by column slices: a block owns 32 vectors (512 bytes)
// of every row and first stages that slice of W_r^T for all E experts in shared memory, so
// a router weight is read from L2 once per block instead of once per routed pair.  A warp
// takes two tokens per pass (2k row loads in flight); the terms are added in the order of
// unpermute_sum_kernel, so the two kernels give the same bits.
constexpr int US_THREADS = 256;
constexpr int US_WARPS = US_THREADS / 32;
template <typename T, int KC>
__global__ void __launch_bounds__(US_THREADS) unpermute_sum_router_kernel(
    const uint4 *__restrict__ dx_perm, const int32_t *__restrict__ sop,
    const float *__restrict__ dgate, const float *__restrict__ gate, const int32_t *__restrict__ idx,
    const uint4 *__restrict__ w_rt, bool accumulate, uint4 *__restrict__ dx, int64_t Tn, int k,
    int nv, int E) {
  extern __shared__ uint4 w_slice[];   // [E][32]
  constexpr int N = Vec<T>::N;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int v0 = blockIdx.y * 32;
  const int v = v0 + lane;
  const bool vin = v < nv;             // (nv % 32 != 0 only for bf16 rows of d % 256 == 128)
  // a token pair's metadata, lane j < k holding pair j's: slot, expert, gate, gate gradient;
  // the next pair's is loaded while this pair's rows are in flight
  struct Meta {
    int slot[2], e[2];
    float g[2], dg[2];
  };
  auto load_meta = [&](int64_t t0, Meta &m) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t t = t0 + u < Tn ? t0 + u : t0;
      const bool on = lane < k;
      m.slot[u] = (dx_perm && on) ? sop[t * k + lane] : 0;
      m.e[u] = on ? idx[t * k + lane] : 0;
      m.g[u] = on ? gate[t * k + lane] : 0.f;
      m.dg[u] = on ? dgate[t * k + lane] : 0.f;
    }
  };
  const int64_t stride = (int64_t)gridDim.x * US_WARPS * 2;
  int64_t t0 = ((int64_t)blockIdx.x * US_WARPS + warp) * 2;
  Meta cur{};
  if (t0 < Tn) load_meta(t0, cur);
  for (int i = threadIdx.x; i < E * 32; i += US_THREADS) {
    const int vv = v0 + (i & 31);
    if (vv < nv) w_slice[i] = __ldg(w_rt + (int64_t)(i >> 5) * nv + vv);
  }
  __syncthreads();
  for (; t0 < Tn; t0 += stride) {
    const int nt = t0 + 1 < Tn ? 2 : 1;
    int slot[2][KC], e[2][KC];
    float dz[2][KC];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      // dz_j = g_j (dg_j - sum_i g_i dg_i), the sum in i order (as token_dz)
      float g[KC], dg[KC], inner = 0.f;
#pragma unroll
      for (int j = 0; j < KC; ++j) {
        slot[u][j] = __shfl_sync(0xffffffffu, cur.slot[u], j);
        e[u][j] = __shfl_sync(0xffffffffu, cur.e[u], j);
        g[j] = __shfl_sync(0xffffffffu, cur.g[u], j);
        dg[j] = __shfl_sync(0xffffffffu, cur.dg[u], j);
        if (j < k) inner = fmaf(g[j], dg[j], inner);
      }
#pragma unroll
      for (int j = 0; j < KC; ++j) dz[u][j] = (j < k) ? g[j] * (dg[j] - inner) : 0.f;
    }
    float acc[2][N];
    uint4 raw[2][KC];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (vin && u < nt && accumulate) {
        Vec<T>::load(dx[(t0 + u) * nv + v], acc[u]);
      } else {
#pragma unroll
        for (int i = 0; i < N; ++i) acc[u][i] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < KC; ++j)
        raw[u][j] = (vin && dx_perm && j < k && u < nt) ? __ldg(dx_perm + (int64_t)slot[u][j] * nv + v)
                                                        : make_uint4(0, 0, 0, 0);
    }
    if (t0 + stride < Tn) load_meta(t0 + stride, cur);
    if (!vin) continue;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (u >= nt) break;
#pragma unroll
      for (int j = 0; j < KC; ++j) {
        if (j < k) {
          float f[N];
          if (dx_perm) {
            Vec<T>::load(raw[u][j], f);
#pragma unroll
            for (int i = 0; i < N; ++i) acc[u][i] += f[i];
          }
          Vec<T>::load(w_slice[e[u][j] * 32 + lane], f);
#pragma unroll
          for (int i = 0; i < N; ++i) acc[u][i] = fmaf(dz[u][j], f[i], acc[u][i]);
        }
      }
      dx[(t0 + u) * nv + v] = Vec<T>::store(acc[u]);
    }
  }
}

template <typename T, int KC>
static cudaError_t launch_unpermute_sum_router(const uint4 *a, const int32_t *sop, const float *dgate,
                                               const float *gate, const int32_t *idx, const uint4 *w,
                                               bool accumulate, uint4 *o, int64_t T_, int k, int nv, int E,
                                               cudaStream_t st) {
  // column slices of 32 vectors; enough token groups to fill every SM at the occupancy the
  // staged W_r^T slice ([E][512 bytes]) allows
  const int nslices = (nv + 31) / 32;
  const int smem = E * 32 * 16;
  auto kern = unpermute_sum_router_kernel<T, KC>;
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  // resident blocks per SM at this E (registers and the staged slice decide), cached per E
  static std::atomic<int> occ_cache[MAX_E + 1];
  int per_sm = occ_cache[E].load(std::memory_order_relaxed);
  if (per_sm <= 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, US_THREADS, smem) != cudaSuccess || per_sm <= 0)
      per_sm = 1;
    occ_cache[E].store(per_sm, std::memory_order_relaxed);
  }
  const int64_t pairs = (T_ + 1) / 2;
  const int64_t gx = std::max<int64_t>(1, std::min<int64_t>((device_sm_count() * per_sm + nslices - 1) / nslices,
                                                            (pairs + US_WARPS - 1) / US_WARPS));
  kern<<<dim3((unsigned)gx, (unsigned)nslices), US_THREADS, smem, st>>>(a, sop, dgate, gate, idx, w, accumulate, o,
                                                                        T_, k, nv, E);
  return cudaGetLastError();
}

// w_rt[e][i] = W_r[i][e] (same storage type), 32x32 tiles through shared memory.
template <typename T>
__global__ void router_transpose_kernel(const T *__restrict__ w_r, T *__restrict__ w_rt, int d,
                                        int E) {
  __shared__ float tile[32][33];
  int i0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    int i = i0 + r, e = e0 + threadIdx.x;
    tile[r][threadIdx.x] = (i < d && e < E) ? to_f(w_r[(int64_t)i * E + e]) : 0.f;
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    int e = e0 + r, i = i0 + threadIdx.x;
    if (e < E && i < d) w_rt[(int64_t)e * d + i] = from_f<T>(tile[threadIdx.x][r]);   // exact
  }
}

// Router weight gradient, stage 1: partial[s][e][c] = sum over tokens of split s of
// dz[t,e] x[t,c].  Thread c owns one column: no atomics, fixed summation order.
constexpr int RW_COLS = 128;
template <typename T>
__global__ void __launch_bounds__(RW_COLS) router_wgrad_partial_kernel(
    const float *__restrict__ dgate, const float *__restrict__ gate, const int32_t *__restrict__ idx,
    const T *__restrict__ x, float *__restrict__ partial, int64_t Tn, int d, int E, int k) {
  extern __shared__ float acc[];  // [E][RW_COLS]
  const int c = blockIdx.x * RW_COLS + threadIdx.x;
  for (int i = threadIdx.x; i < E * RW_COLS; i += RW_COLS) acc[i] = 0.f;
  __syncthreads();
  const int64_t per = (Tn + RB_SPLIT - 1) / RB_SPLIT;
  const int64_t tb = (int64_t)blockIdx.y * per;
  const int64_t te = min(Tn, tb + per);
  if (c < d) {
    for (int64_t t = tb; t < te; ++t) {
      float dz[MAX_K];
      token_dz(dgate, gate, t, k, dz);
      float xv = to_f(x[t * d + c]);
#pragma unroll
      for (int j = 0; j < MAX_K; ++j)
        if (j < k) acc[idx[t * k + j] * RW_COLS + threadIdx.x] += dz[j] * xv;
    }
  }
  __syncthreads();
  float *out = partial + (int64_t)blockIdx.y * E * d;
  if (c < d)
    for (int e = 0; e < E; ++e) out[(int64_t)e * d + c] = acc[e * RW_COLS + threadIdx.x];
}

// Stage 2: dW_r[c][e] = sum_s partial[s][e][c], in split order.
__global__ void router_wgrad_reduce_kernel(const float *__restrict__ partial, float *__restrict__ dw_r,
                                           int d, int E) {
  int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= (int64_t)d * E) return;
  int e = (int)(n / d), c = (int)(n % d);
  float s = 0.f;
  for (int sp = 0; sp < RB_SPLIT; ++sp) s += partial[(int64_t)sp * E * d + n];
  dw_r[(int64_t)c * E + e] = s;
}

// dst[b][c][r] = src[b][r][c], 32x32 tiles through shared memory.
__global__ void transpose_batched_kernel(const float *__restrict__ src, float *__restrict__ dst, int R,
                                         int C) {
  __shared__ float tile[32][33];
  const int64_t b = blockIdx.z;
  const float *s = src + b * R * C;
  float *d = dst + b * R * C;
  int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    int r = r0 + i, c = c0 + threadIdx.x;
    if (r < R && c < C) tile[i][threadIdx.x] = s[(int64_t)r * C + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    int c = c0 + i, r = r0 + threadIdx.x;
    if (r < R && c < C) d[(int64_t)c * R + r] = tile[threadIdx.x][i];
  }
}

cudaError_t launch_transpose_batched(const float *src, float *dst, int B, int R, int C, cudaStream_t st) {
  dim3 grid((C + 31) / 32, (R + 31) / 32, B), block(32, 8);
  transpose_batched_kernel<<<grid, block, 0, st>>>(src, dst, R, C);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// Router weight gradient from the expert-contiguous rows (layer backward):
//   dW_r[c][e] = sum over slots s of expert e of dz(s) * x_perm[s][c],
// where dz(s) is the logit gradient of the pair in slot s.  The rows of every expert are
// cut into chunks of RG_ROWS; chunk q covers rows of one expert only, so its partial sum
// belongs to that expert; a second kernel adds an expert's chunks in order.
// ---------------------------------------------------------------------------------------
constexpr int RG_ROWS = 64;
constexpr int RG_THREADS = 128;  // x one 16-byte vector each

// dz_slot[s] = g (dg - sum_j' g_j' dg_j') of the pair in slot s
__global__ void router_dz_slot_kernel(const int32_t *__restrict__ pos, const float *__restrict__ dgate,
                                      const float *__restrict__ gate, float *__restrict__ dz_slot,
                                      int64_t P, int k) {
  int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= P) return;
  int64_t p = pos[s];
  int64_t t = p / k;
  float inner = 0.f;
  for (int j = 0; j < k; ++j) inner = fmaf(gate[t * k + j], dgate[t * k + j], inner);
  dz_slot[s] = gate[p] * (dgate[p] - inner);
}

// Exclusive prefix over experts of ceil(count_e / RG_ROWS), one warp; returns the total.
__device__ int chunk_prefix(const int32_t *offsets, int E, int *prefix) {
  const int lane = threadIdx.x & 31;
  int cnt[8], sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int e = lane * 8 + i;
    cnt[i] = (e < E) ? (offsets[e + 1] - offsets[e] + RG_ROWS - 1) / RG_ROWS : 0;
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
    if (e < E) prefix[e] = run;
    run += cnt[i];
  }
  if (lane == 31) prefix[E] = incl;
  return __shfl_sync(0xffffffffu, incl, 31);
}

// x_perm rows in slot order, or (pos != nullptr) the layer input's rows x[pos[slot] / k].
// Thread v owns one 16-byte vector (8 bf16 or 4 fp32 columns) of the rows; each column's
// sum runs over the chunk's rows in order.
template <typename T>
__global__ void __launch_bounds__(RG_THREADS) router_wgrad_grouped_kernel(
    const uint4 *__restrict__ x_perm, const float *__restrict__ dz_slot, const int32_t *__restrict__ offsets,
    float *__restrict__ partial, int E, int d, const int32_t *__restrict__ pos, int k) {
  constexpr int N = Vec<T>::N;
  __shared__ int prefix[MAX_E + 1];
  if (threadIdx.x < 32) chunk_prefix(offsets, E, prefix);
  __syncthreads();
  const int q = blockIdx.x;
  if (q >= prefix[E]) return;
  int lo = 0, hi = E;  // prefix[lo] <= q < prefix[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (prefix[mid] <= q) lo = mid; else hi = mid;
  }
  const int e = lo;
  const int r0 = offsets[e] + (q - prefix[e]) * RG_ROWS;
  const int r1 = min(offsets[e + 1], r0 + RG_ROWS);
  const int nv = d / N;
  const int v = blockIdx.y * RG_THREADS + threadIdx.x;
  if (v >= nv) return;
  auto row_of = [&](int slot) -> int64_t { return pos ? (int64_t)(pos[slot] / k) : (int64_t)slot; };
  float a[N];
#pragma unroll
  for (int i = 0; i < N; ++i) a[i] = 0.f;
  int r = r0;
  for (; r + 4 <= r1; r += 4) {
    float z[4];
    uint4 raw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      z[u] = dz_slot[r + u];
      raw[u] = __ldg(x_perm + row_of(r + u) * nv + v);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float f[N];
      Vec<T>::load(raw[u], f);
#pragma unroll
      for (int i = 0; i < N; ++i) a[i] = fmaf(z[u], f[i], a[i]);
    }
  }
  for (; r < r1; ++r) {
    const float z = dz_slot[r];
    float f[N];
    Vec<T>::load(__ldg(x_perm + row_of(r) * nv + v), f);
#pragma unroll
    for (int i = 0; i < N; ++i) a[i] = fmaf(z, f[i], a[i]);
  }
  float4 *out = reinterpret_cast<float4 *>(partial + (int64_t)q * d + (int64_t)v * N);
#pragma unroll
  for (int i = 0; i < N; i += 4) out[i / 4] = make_float4(a[i], a[i + 1], a[i + 2], a[i + 3]);
}

// dW_r[c][e] = sum of expert e's chunk partials, in chunk order (0 for an empty expert).
__global__ void router_wgrad_grouped_reduce_kernel(const float *__restrict__ partial,
                                                   const int32_t *__restrict__ offsets,
                                                   float *__restrict__ dw_r, int E, int d) {
  __shared__ int prefix[MAX_E + 1];
  if (threadIdx.x < 32) chunk_prefix(offsets, E, prefix);
  __syncthreads();
  const int e = blockIdx.y;
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= d) return;
  float s = 0.f;
  for (int q = prefix[e]; q < prefix[e + 1]; ++q) s += partial[(int64_t)q * d + c];
  dw_r[(int64_t)c * E + e] = s;
}

cudaError_t launch_router_wgrad_grouped(const Shape &s, const void *x_perm, const int32_t *pos,
                                        const int32_t *offsets, const float *dgate, const float *gate,
                                        float *dz_slot, float *partial, float *dw_r, cudaStream_t st,
                                        const void *x) {
  const void *rows = x ? x : x_perm;
  const int32_t *rpos = x ? pos : nullptr;
  const int64_t P = s.P();
  router_dz_slot_kernel<<<(unsigned)((P + 255) / 256), 256, 0, st>>>(pos, dgate, gate, dz_slot, P, s.k);
  const int64_t max_chunks = (P + RG_ROWS - 1) / RG_ROWS + s.E;
  const int nv = s.d * s.es() / 16;
  dim3 grid((unsigned)max_chunks, (unsigned)((nv + RG_THREADS - 1) / RG_THREADS));
  if (s.dtype == MOE_BF16)
    router_wgrad_grouped_kernel<bf16><<<grid, RG_THREADS, 0, st>>>(static_cast<const uint4 *>(rows), dz_slot,
                                                                   offsets, partial, s.E, s.d, rpos, s.k);
  else
    router_wgrad_grouped_kernel<float><<<grid, RG_THREADS, 0, st>>>(static_cast<const uint4 *>(rows), dz_slot,
                                                                    offsets, partial, s.E, s.d, rpos, s.k);
  dim3 g2((unsigned)((s.d + 255) / 256), (unsigned)s.E);
  router_wgrad_grouped_reduce_kernel<<<g2, 256, 0, st>>>(partial, offsets, dw_r, s.E, s.d);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// Tail buffers of the bf16 weight-gradient GEMMs, which reduce over each expert's rows in
// K-blocks of 64: the expert's last, partial block is copied into its own 64 rows with zeros
// after the expert's rows, so that the GEMM loads it like any other block.  The GEMM reads
// only the 16-row slices that hold expert rows, so rows from the next multiple of 16 on are
// left as they are.  One block per (row i of the tail, expert e, operand: A or B).
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128) wgrad_tail_kernel(const uint4 *__restrict__ src_a, int nv_a,
                                                         uint4 *__restrict__ tails_a,
                                                         const uint4 *__restrict__ src_b, int nv_b,
                                                         uint4 *__restrict__ tails_b,
                                                         const int32_t *__restrict__ offsets) {
  const int i = blockIdx.x, e = blockIdx.y;
  const int lo = offsets[e], cnt = offsets[e + 1] - lo;
  const int full = cnt / WGRAD_TAIL_ROWS * WGRAD_TAIL_ROWS, v = cnt - full;
  if (v == 0 || i >= (v + 15) / 16 * 16) return;   // rows the GEMM never reads
  const bool b = blockIdx.z == 1;
  const uint4 *src = b ? src_b : src_a;
  const int nv = b ? nv_b : nv_a;
  uint4 *dst = (b ? tails_b : tails_a) + ((int64_t)e * WGRAD_TAIL_ROWS + i) * nv;
  if (i < v) {
    const uint4 *row = src + ((int64_t)lo + full + i) * nv;
    for (int c = threadIdx.x; c < nv; c += 128) dst[c] = __ldg(row + c);
  } else {
    for (int c = threadIdx.x; c < nv; c += 128) dst[c] = make_uint4(0, 0, 0, 0);
  }
}

cudaError_t launch_wgrad_tails(const void *src_a, int C_a, void *tails_a, const void *src_b, int C_b, void *tails_b,
                               const int32_t *offsets, int E, cudaStream_t st) {
  dim3 grid(WGRAD_TAIL_ROWS, (unsigned)E, 2);
  wgrad_tail_kernel<<<grid, 128, 0, st>>>(static_cast<const uint4 *>(src_a), C_a * 2 / 16,
                                          static_cast<uint4 *>(tails_a), static_cast<const uint4 *>(src_b),
                                          C_b * 2 / 16, static_cast<uint4 *>(tails_b), offsets);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------ launchers
static unsigned row_grid(int64_t T) { return (unsigned)((T + ROW_WARPS - 1) / ROW_WARPS); }

cudaError_t launch_permute(const Shape &s, const void *x, const int32_t *sop, void *x_perm,
                           cudaStream_t st) {
  if (s.T == 0) return cudaSuccess;
  int nv = s.d * s.es() / 16;
  permute_kernel<<<row_grid(s.T), ROW_THREADS, 0, st>>>(static_cast<const uint4 *>(x), sop,
                                                        static_cast<uint4 *>(x_perm), s.T, s.k, nv);
  return cudaGetLastError();
}

cudaError_t launch_unpermute_combine(const Shape &s, const void *y_perm, const int32_t *sop,
                                     const float *gate, void *y, cudaStream_t st, bool accumulate) {
  if (s.T == 0) return cudaSuccess;
  int nv = s.d * s.es() / 16;
  auto yp = static_cast<const uint4 *>(y_perm);
  auto yo = static_cast<uint4 *>(y);
  const dim3 grid(row_grid(s.T));
  if (s.dtype == MOE_BF16) {
    if (s.k <= 4) combine_kernel<bf16, 4><<<grid, ROW_THREADS, 0, st>>>(yp, sop, gate, yo, s.T, s.k, nv, accumulate);
    else combine_kernel<bf16, MAX_K><<<grid, ROW_THREADS, 0, st>>>(yp, sop, gate, yo, s.T, s.k, nv, accumulate);
  } else {
    if (s.k <= 4) combine_kernel<float, 4><<<grid, ROW_THREADS, 0, st>>>(yp, sop, gate, yo, s.T, s.k, nv, accumulate);
    else combine_kernel<float, MAX_K><<<grid, ROW_THREADS, 0, st>>>(yp, sop, gate, yo, s.T, s.k, nv, accumulate);
  }
  return cudaGetLastError();
}

// offsets of one group holding every token: {0, T}
__global__ void group_offsets_kernel(int32_t *o, int32_t T) {
  if (threadIdx.x == 0) {
    o[0] = 0;
    o[1] = T;
  }
}

cudaError_t launch_group_offsets(int32_t *o, int64_t T, cudaStream_t st) {
  group_offsets_kernel<<<1, 32, 0, st>>>(o, (int32_t)T);
  return cudaGetLastError();
}

cudaError_t launch_combine_bwd(const Shape &s, const void *dy, const void *y_perm, const int32_t *sop,
                               const float *gate, void *dy_perm, float *dgate, cudaStream_t st) {
  if (s.T == 0) return cudaSuccess;
  int nv = s.d * s.es() / 16;
  auto a = static_cast<const uint4 *>(dy);
  auto b = static_cast<const uint4 *>(y_perm);
  auto o = static_cast<uint4 *>(dy_perm);
  if (s.dtype == MOE_BF16)
    combine_bwd_kernel<bf16><<<row_grid(s.T), ROW_THREADS, 0, st>>>(a, b, sop, gate, o, dgate, s.T, s.k, nv);
  else
    combine_bwd_kernel<float><<<row_grid(s.T), ROW_THREADS, 0, st>>>(a, b, sop, gate, o, dgate, s.T, s.k, nv);
  return cudaGetLastError();
}

cudaError_t launch_unpermute_sum(const Shape &s, const void *dx_perm, const int32_t *sop,
                                 const float *dgate, const float *gate, const int32_t *idx,
                                 const void *w_rt, bool accumulate, void *dx, cudaStream_t st) {
  if (s.T == 0) return cudaSuccess;
  int nv = s.d * s.es() / 16;
  auto a = static_cast<const uint4 *>(dx_perm);
  auto w = static_cast<const uint4 *>(w_rt);
  auto o = static_cast<uint4 *>(dx);
  if (w) {
    if (s.dtype == MOE_BF16)
      return s.k <= 4 ? launch_unpermute_sum_router<bf16, 4>(a, sop, dgate, gate, idx, w, accumulate, o, s.T, s.k,
                                                              nv, s.E, st)
                      : launch_unpermute_sum_router<bf16, MAX_K>(a, sop, dgate, gate, idx, w, accumulate, o, s.T,
                                                                 s.k, nv, s.E, st);
    return s.k <= 4 ? launch_unpermute_sum_router<float, 4>(a, sop, dgate, gate, idx, w, accumulate, o, s.T, s.k, nv,
                                                             s.E, st)
                    : launch_unpermute_sum_router<float, MAX_K>(a, sop, dgate, gate, idx, w, accumulate, o, s.T,
                                                                s.k, nv, s.E, st);
  }
  if (s.dtype == MOE_BF16)
    unpermute_sum_kernel<bf16><<<row_grid(s.T), ROW_THREADS, 0, st>>>(a, sop, dgate, gate, idx, w,
                                                                      accumulate, o, s.T, s.k, nv);
  else
    unpermute_sum_kernel<float><<<row_grid(s.T), ROW_THREADS, 0, st>>>(a, sop, dgate, gate, idx, w,
                                                                       accumulate, o, s.T, s.k, nv);
  return cudaGetLastError();
}

cudaError_t launch_router_transpose(const Shape &s, const void *w_r, void *w_rt, cudaStream_t st) {
  dim3 grid((s.d + 31) / 32, (s.E + 31) / 32), block(32, 8);
  if (s.dtype == MOE_BF16)
    router_transpose_kernel<bf16><<<grid, block, 0, st>>>(static_cast<const bf16 *>(w_r), static_cast<bf16 *>(w_rt),
                                                          s.d, s.E);
  else
    router_transpose_kernel<float><<<grid, block, 0, st>>>(static_cast<const float *>(w_r),
                                                           static_cast<float *>(w_rt), s.d, s.E);
  return cudaGetLastError();
}

cudaError_t launch_router_wgrad(const Shape &s, const float *dgate, const float *gate,
                                const int32_t *idx, const void *x, float *partial, float *dw_r,
                                cudaStream_t st) {
  size_t smem = (size_t)s.E * RW_COLS * sizeof(float);
  dim3 grid((s.d + RW_COLS - 1) / RW_COLS, RB_SPLIT);
  cudaError_t e;
  if (s.dtype == MOE_BF16) {
    e = cudaFuncSetAttribute(router_wgrad_partial_kernel<bf16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    router_wgrad_partial_kernel<bf16><<<grid, RW_COLS, smem, st>>>(
        dgate, gate, idx, static_cast<const bf16 *>(x), partial, s.T, s.d, s.E, s.k);
  } else {
    e = cudaFuncSetAttribute(router_wgrad_partial_kernel<float>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    router_wgrad_partial_kernel<float><<<grid, RW_COLS, smem, st>>>(
        dgate, gate, idx, static_cast<const float *>(x), partial, s.T, s.d, s.E, s.k);
  }
  int64_t n = (int64_t)s.d * s.E;
  router_wgrad_reduce_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(partial, dw_r, s.d, s.E);
  return cudaGetLastError();
}

}  // namespace moe
