// Grouped SwiGLU expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Method: unite.ai "Ai2 κυκλοφορεί το Olmo-Core 3 ...", section "Παραλληλισμός,
// Ακρίβεια και Τεχνικές Μνήμης": a grouped GEMM runs the experts' many small matmuls
// together, with the matmuls scheduled from the device so that nothing waits on the
// host; ettayeb.fr "Olmo-core 3 ouvre l'entraînement des MoE ...", section "Trois
// parallélismes, trois optimisations de routage"; bigchange.ai "Olmo-core 3 открывает
// стек обучения MoE от Ai2 ...", section "Три числа, три знаменателя" (the gains sit in
// the feed-forward compute).
//
// One persistent kernel, one CTA per SM, 10 warps:
//   warp 0      TMA producer: fills a STAGES-deep ring of (A, B) K-blocks in shared
//               memory (128-byte swizzle), one mbarrier per stage;
//   warp 1      allocates TMEM; its lane 0 issues tcgen05.mma (128 x BN x 16 per
//               instruction) into one of two TMEM accumulators and commits each stage
//               back to the producer;
//   warps 2..9  epilogue: tcgen05.ld the accumulator (warp w reads TMEM lanes
//               32*(w%4)..+31, i.e. one row per thread; two warps per lane quarter split
//               the columns), apply the fused elementwise step and store to global
//               memory (weight gradients: through shared memory and TMA stores), then
//               release the accumulator;
// The epilogue of tile i overlaps the MMAs of tile i+1 (double-buffered accumulator).
//
// Tile schedule.  Row-grouped GEMMs (forward and data-gradient) tile every expert's row
// range [offsets[e], offsets[e+1]) in 128-row blocks; each CTA rebuilds the per-expert
// block prefix from `offsets` on the device, so the host never learns the counts.
// Rows of a block that belong to the next expert are computed and not stored.
// Weight-gradient GEMMs reduce over one expert's rows; the expert's last, partial K-block is
// read from a per-expert tail buffer that holds its rows and zeros after them (bf16; the
// MXFP8 operands are padded to 128 rows per expert instead), so every stage is an ordinary
// load.  bf16 weight gradients deal whole strips (one expert's M block: all N tiles that
// share the A operand) to the CTAs (pairs) and keep A's K-blocks resident in shared memory
// across the strip, so that only B streams through the ring (A stationary); an expert whose
// K-blocks outnumber the A slots streams A with B instead.
// CTA pairs (cta_group::2): a 256-row tile whose MMAs the even CTA issues for both.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "common.cuh"
#include "mxfp8.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace gg {

enum Mode { FWD_GU = 0, FWD_DOWN = 1, DGRAD_DOWN = 2, DGRAD_GU = 3, WGRAD_DOWN = 4, WGRAD_GU = 5, ROUTER = 6 };

constexpr int BM = 128;
constexpr int EPI_WARPS = 8;
constexpr int NUM_THREADS = 32 * (2 + EPI_WARPS);  // producer, MMA issuer, epilogue warps
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s: far above any tile's time

template <int MODE> struct ModeTraits {
  static constexpr bool A_MN = (MODE == WGRAD_DOWN || MODE == WGRAD_GU);
  static constexpr bool B_MN = (MODE == FWD_GU || MODE == FWD_DOWN || MODE == WGRAD_DOWN || MODE == WGRAD_GU ||
                                MODE == ROUTER);
  static constexpr bool WGRAD = A_MN;
};

// MXFP8 operand tag: E4M3 codes with E8M0 scales per 32 K-elements (outputs stay bf16).
struct e4m3 {
  uint8_t v;
};

template <typename T> struct ElemTraits;
template <> struct ElemTraits<bf16> {
  static constexpr int ES = 2;
  static constexpr uint32_t FMT = 1;  // BF16 in the instruction descriptor
  using Out = bf16;
};
template <> struct ElemTraits<float> {
  static constexpr int ES = 4;
  static constexpr uint32_t FMT = 2;  // TF32
  using Out = float;
};
template <> struct ElemTraits<e4m3> {
  static constexpr int ES = 1;
  static constexpr uint32_t FMT = 0;  // E4M3 in the block-scaled instruction descriptor
  using Out = bf16;
};

constexpr int SMEM_LIMIT = 227 * 1024;
constexpr int CTRL_BYTES = 2048;

// BN: the MMA's N.  CG: CTAs per MMA (1, or 2 for a 256-row pair tile in which each CTA
// holds 128 rows of A and BN/2 columns of B).  EXTRA: bytes of shared memory the mode keeps
// after the control block; the stage ring gives way to them.
template <typename T, int BN, int CG = 1, int EXTRA = 0> struct Cfg {
  static constexpr bool MX = (ElemTraits<T>::ES == 1);
  static constexpr int BMP = BM * CG;                   // rows of an MMA tile (pair)
  static constexpr int BNC = BN / CG;                   // columns of B held by one CTA
  static constexpr int ES = ElemTraits<T>::ES;
  static constexpr int KBLK = 128 / ES;                 // K elements per stage (one 128-B swizzle row)
  static constexpr int UMMA_K = 32 / ES;                // K per tcgen05.mma
  static constexpr int BOX_MN = 128 / ES;               // MN elements per TMA box of an MN-major operand
  static constexpr int BOX_BYTES = KBLK * 128;          // bytes of one [KBLK x BOX_MN] box
  static constexpr int A_BYTES = BM * KBLK * ES;
  static constexpr int B_BYTES = BNC * KBLK * ES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // two accumulators; MXFP8 adds 8 columns of scale factors (A: 4, B: 4) after them
  static constexpr int TMEM_COLS = MX ? 512 : 2 * BN;
  static constexpr int SF_BYTES = MX ? 1024 : 0;        // per stage: 512-byte scale blocks of A and B
  static constexpr int STAGES_WANTED = (STAGE_BYTES >= 48 * 1024) ? 4 : (STAGE_BYTES >= 32 * 1024 ? 6 : 8);
  static constexpr int STAGES_FIT = (SMEM_LIMIT - 1024 - CTRL_BYTES - EXTRA) / (STAGE_BYTES + SF_BYTES);
  static constexpr int STAGES = STAGES_WANTED < STAGES_FIT ? STAGES_WANTED : STAGES_FIT;
  static_assert(STAGES >= 2, "shared memory");
  static constexpr int SMEM_BYTES = STAGES * (STAGE_BYTES + SF_BYTES) + 1024 /*align slack*/ + CTRL_BYTES + EXTRA;
};

struct Params {
  const int32_t *offsets;
  int E;
  int P;       // rows of the row-grouped tensors
  int K;       // reduction length (row-grouped modes)
  int N;       // output columns
  int M;       // output rows per expert (weight-gradient modes)
  int f, d;
  void *out0;
  void *out1;
  void *out2;
  const void *aux;
  int k;       // router: experts per token
  // MXFP8 scale factors in the tile layout the quantisers write (tiles of 128 M or N indices
  // by 4 K-blocks, 512 bytes, in the arrangement of tcgen05.cp's 32x128b.warpx4 copy); the
  // tile of (MN block b, K group g) is at (b * nk + g) * 512, nk = the operand's K extent in
  // groups of 128 elements
  const uint8_t *sfa;
  const uint8_t *sfb;
  int nka, nkb;
  // MXFP8 epilogues that quantise their own bf16 output for the next GEMMs (nullptr: none),
  // rows padded to 128 per expert as the row-grouped MXFP8 GEMMs index them, scales in the
  // tile layout: q_row* blocks of 32 along the row (nk_row = K groups of a row), q_col*
  // blocks of 32 down the rows (nk_col = K groups of the padded token axis)
  uint8_t *q_row_codes, *q_row_scales, *q_col_codes, *q_col_scales;
  int nk_row, nk_col;
  // bf16 weight gradients (A stationary): na of the ring's slots hold A, the rest are B's
  // ring; strips: tiles are dealt in whole strips that keep A resident (else tile by tile,
  // A streaming with B)
  int na, strips;
  int *err;
  int *where;  // [3]: first failed wait per role, ((tile+1) << 12) | (kb << 2) | site
  // Failure-detection test hook, 0 in normal use: the MMA issuer of a single-CTA launch first
  // waits up to stall_ns on a barrier nothing arrives on, so that the wait runs out and the
  // kernel takes its abort path (every role stops, in-flight copies and MMAs are drained,
  // MOE_ERR_DEVICE_TIMEOUT is reported).
  uint64_t stall_ns;
};

__device__ __forceinline__ void note_fail(const Params &p, int role, int t, int kb, int site) {
  if (p.where) atomicCAS(&p.where[role], 0, ((t + 1) << 12) | ((kb & 0x3FF) << 2) | (site & 3));
}

struct Tile {
  int e, m_blk, n_blk;
  int orow0;      // first output row (row-grouped modes)
  int mcol0;      // weight-gradient modes: first M index (A column, output row) of this CTA
  int row0;       // first A row (row-grouped) or first K row (weight-gradient)
  int rows;       // valid rows (row-grouped) or valid K rows (weight-gradient)
  int num_kb;
};

// Shared control block placed after the stage ring.
struct Ctrl {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t afull[8];      // A-stationary weight gradients: one pair of barriers per A slot
  uint64_t aempty[8];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint64_t never;         // the failure-detection hook's barrier: nothing ever arrives on it
  uint64_t xfull[4];      // router: one lane quarter's second-half picks are in xbuf
  uint64_t xempty[4];     // router: ... and have been merged
  uint32_t tmem_base;
  int abort;
  int strips;             // A-stationary weight gradients: every expert's A fits its slots
  union {
    int prefix[MAX_E + 1];  // exclusive prefix of 128-row blocks per expert
    float bias[MAX_E];      // router: the logit bias (0 past E)
    int offs[MAX_E + 1];    // bf16 weight gradients: a copy of offsets (prefix is unused there)
  };
};
static_assert(sizeof(Ctrl) <= CTRL_BYTES, "control block");
// Router: shared buffer for the second-half picks, [MAX_K][BM] keys then [MAX_K][BM] experts
constexpr int ROUTER_XBYTES = 2 * MAX_K * BM * 4;
// Weight gradients: each epilogue warp stages its output in one box of 32 rows x 64 bf16
// columns (128-byte rows, 128-byte swizzle) that TMA stores write out.  One box per warp
// (32 KB in all) leaves room for six pipeline stages of 32 KB.
constexpr int EPI_BOX_BYTES = 32 * 128;
constexpr int WGRAD_XBYTES = EPI_WARPS * EPI_BOX_BYTES;
// Row-grouped GEMMs: a copy of offsets [E+1] after the control block, read by every role's
// tile lookup (one global load per tile per role otherwise, on the MMA issuer's critical path).
constexpr int OFFS_BYTES = 1152;
template <int MODE> constexpr int extra_smem() {
  return MODE == ROUTER ? ROUTER_XBYTES : ModeTraits<MODE>::WGRAD ? WGRAD_XBYTES : OFFS_BYTES;
}

// offs: offsets [E+1] (a shared-memory copy where the kernel keeps one)
template <int MODE, int BN, int KBLK, bool MX, int CG = 1>
__device__ __forceinline__ bool get_tile(int t, const Params &p, const Ctrl &c, const int *offs, Tile &tl,
                                         int rank = 0) {
  constexpr int BMP = BM * CG;
  if constexpr (MODE == ROUTER) {
    tl.e = 0;
    tl.m_blk = t;
    tl.n_blk = 0;
    tl.row0 = tl.orow0 = t * BM;
    tl.rows = min(BM, p.P - t * BM);
    tl.num_kb = p.K / KBLK;
  } else if constexpr (ModeTraits<MODE>::WGRAD) {
    const int mt = p.M / BMP, nt = p.N / BN;
    tl.e = t / (mt * nt);
    int r = t - tl.e * mt * nt;
    tl.m_blk = r / nt;
    tl.n_blk = r - tl.m_blk * nt;
    tl.mcol0 = tl.m_blk * BMP + rank * BM;
    int lo = offs[tl.e], hi = offs[tl.e + 1];
    tl.rows = hi - lo;
    if constexpr (MX) {
      // quantised operands live in expert buffers padded to 128 rows (zeros past the end)
      tl.row0 = c.prefix[tl.e] * BM;
      tl.num_kb = c.prefix[tl.e + 1] - c.prefix[tl.e];
    } else {
      tl.row0 = lo;
      tl.num_kb = (tl.rows + KBLK - 1) / KBLK;
    }
    tl.orow0 = 0;
  } else {
    const int nt = p.N / BN;
    int g = t / nt;
    tl.n_blk = t - g * nt;
    // largest e with prefix[e] <= g (prefix is non-decreasing, prefix[0] = 0)
    int lo = 0, hi = p.E;  // invariant: prefix[lo] <= g < prefix[hi]
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (c.prefix[mid] <= g) lo = mid; else hi = mid;
    }
    tl.e = lo;
    tl.m_blk = g - c.prefix[lo];
    int off = offs[lo], cnt = offs[lo + 1] - off;
    tl.orow0 = off + tl.m_blk * BMP + rank * BM;   // this CTA's rows of the (pair) tile
    tl.row0 = MX ? g * BM : tl.orow0;   // quantised A: expert buffers padded to 128 rows
    tl.rows = min(BM, cnt - tl.m_blk * BMP - rank * BM);   // may be <= 0 for the second CTA
    tl.mcol0 = 0;
    tl.num_kb = p.K / KBLK;
  }
  return true;
}

// The i-th tile of this CTA (pair), or -1 past the last.  strips: strip s = tile0 + j*tstep
// holds tiles s*nt .. s*nt + nt-1 (nt = N/BN, the tiles that share one A block).
template <int BN>
__device__ __forceinline__ int nth_tile(int i, const Params &p, int tile0, int tstep, int ntiles, bool strips) {
  int t;
  if (strips) {
    const int nt = p.N / BN;
    t = (tile0 + (i / nt) * tstep) * nt + i % nt;
  } else {
    t = tile0 + i * tstep;
  }
  return t < ntiles ? t : -1;
}

template <int MODE, int BN, int CG = 1>
__device__ __forceinline__ int total_tiles(const Params &p, const Ctrl &c) {
  if constexpr (MODE == ROUTER) return (p.P + BM - 1) / BM;
  else if constexpr (ModeTraits<MODE>::WGRAD) return p.E * (p.M / (BM * CG)) * (p.N / BN);
  else return c.prefix[p.E] * (p.N / BN);
}

// Store 32 consecutive values of one row.
template <typename T>
__device__ __forceinline__ void store32(T *dst, const float (&v)[32]) {
  uint4 *d4 = reinterpret_cast<uint4 *>(dst);
  constexpr int N = Vec<T>::N;
#pragma unroll
  for (int i = 0; i < 32 / N; ++i) d4[i] = Vec<T>::store(&v[i * N]);
}
__device__ __forceinline__ uint4 shfl_xor4(uint4 v, int m) {
  v.x = __shfl_xor_sync(0xffffffffu, v.x, m);
  v.y = __shfl_xor_sync(0xffffffffu, v.y, m);
  v.z = __shfl_xor_sync(0xffffffffu, v.z, m);
  v.w = __shfl_xor_sync(0xffffffffu, v.w, m);
  return v;
}

// Store a 32-row x 32-column slab held one row per lane (lane l: slab row l, values v).
// dst points at column 0 of slab row 0; ld is the row stride in elements; rows >= nvalid
// are not written.  Every lane of the warp must call it.
// bf16: a 4x4 transpose of 16-byte pieces inside each group of four lanes, so that each
// store instruction writes eight whole 64-byte row segments instead of 32 scattered
// 16-byte pieces.  fp32: each lane writes its own row.
template <typename T>
__device__ __forceinline__ void store_slab(T *dst, int64_t ld, int nvalid, const float (&v)[32]) {
  const int lane = threadIdx.x & 31;
  if constexpr (sizeof(T) == 2) {
    uint4 q[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) q[c] = Vec<T>::store(&v[8 * c]);
    const int j = lane & 3;
    {  // exchange with lane ^ 1: 1x1 blocks
      const bool odd = j & 1;
      uint4 r0 = shfl_xor4(odd ? q[0] : q[1], 1);
      uint4 r1 = shfl_xor4(odd ? q[2] : q[3], 1);
      if (odd) { q[0] = r0; q[2] = r1; } else { q[1] = r0; q[3] = r1; }
    }
    {  // exchange with lane ^ 2: 2x2 blocks
      const bool hi = j & 2;
      uint4 r0 = shfl_xor4(hi ? q[0] : q[2], 2);
      uint4 r1 = shfl_xor4(hi ? q[1] : q[3], 2);
      if (hi) { q[0] = r0; q[1] = r1; } else { q[2] = r0; q[3] = r1; }
    }
    // lane (4g + j) now holds piece j of slab rows 4g + 0..3
    const int g4 = lane & ~3;
#pragma unroll
    for (int s2 = 0; s2 < 4; ++s2)
      if (g4 + s2 < nvalid) reinterpret_cast<uint4 *>(dst + (int64_t)(g4 + s2) * ld)[j] = q[s2];
  } else {
    if (lane < nvalid) store32(dst + (int64_t)lane * ld, v);
  }
}

template <typename T>
__device__ __forceinline__ void load32(const T *src, float (&v)[32]) {
  const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
  constexpr int N = Vec<T>::N;
#pragma unroll
  for (int i = 0; i < 32 / N; ++i) Vec<T>::load(s4[i], &v[i * N]);
}

__device__ __forceinline__ float sigmoidf_(float h) { return 1.0f / (1.0f + __expf(-h)); }

// Router order key: an unsigned 32-bit number that grows with the logit (-0 counts as +0),
// 1 for NaN (below every number) and 0 for "no expert".  Among equal keys the lower expert
// index ranks first.
__device__ __forceinline__ uint32_t router_key(float z) {
  if (z != z) return 1u;
  const uint32_t b = __float_as_uint(z == 0.f ? 0.f : z);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float router_key_value(uint32_t o) {
  if (o <= 1u) return __uint_as_float(0x7fc00000u);
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}
// (o, e) ranks above (p, f): the larger key, then the lower expert
__device__ __forceinline__ bool key_above(uint32_t o, int e, uint32_t po, int pe) {
  return o > po || (o == po && e < pe);
}

template <typename T, int BN, int MODE, int CG>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1,
                        const __grid_constant__ CUtensorMap tmO0,   // weight gradients: outputs
                        const __grid_constant__ CUtensorMap tmO1,
                        const __grid_constant__ CUtensorMap tmAT,   // bf16 weight gradients: tail
                        const __grid_constant__ CUtensorMap tmBT,   // buffers of A and B
                        const Params p) {
  using C = Cfg<T, BN, CG, extra_smem<MODE>()>;
  static_assert(CG == 1 || (sizeof(T) == 2 && MODE != ROUTER), "CTA pairs: bf16 grouped GEMMs only");
  constexpr int BMP = C::BMP, BNC = C::BNC;
  using MT = ModeTraits<MODE>;
  // tf32 operands are only ever K-major: the fp32 forward reads pre-transposed weights
  constexpr bool FWD_B_KMAJOR = (sizeof(T) == 4) && (MODE == FWD_GU || MODE == FWD_DOWN);
  constexpr bool B_MN = MT::B_MN && !FWD_B_KMAJOR;
  constexpr bool ASTAT = MT::WGRAD && !C::MX;   // A stationary (bf16 weight gradients), below
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *ring = smem;                                   // STAGES x (A | B)
  uint8_t *sf_ring = smem + C::STAGES * C::STAGE_BYTES;   // MXFP8: STAGES x (SFA | SFB)
  Ctrl &c = *reinterpret_cast<Ctrl *>(smem + C::STAGES * (C::STAGE_BYTES + C::SF_BYTES));
  uint8_t *extra = smem + C::STAGES * (C::STAGE_BYTES + C::SF_BYTES) + CTRL_BYTES;   // 1024-byte aligned
  uint32_t *xbuf = reinterpret_cast<uint32_t *>(extra);
  volatile int *abort_flag = &c.abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA pairs: rank 0 (the leader) issues the MMAs for both CTAs; tiles are dealt per pair
  const int rank = CG == 2 ? (int)ptx::cluster_ctarank() : 0;
  const int tile0 = CG == 2 ? (int)ptx::cluster_id_x() : (int)blockIdx.x;
  const int tstep = CG == 2 ? (int)ptx::ncluster_x() : (int)gridDim.x;

  // ------------------------------------------------------------------ prologue
  if (threadIdx.x == 0) {
    for (int s = 0; s < 8; ++s) {
      // one arrival: the producer's arrive.expect_tx (pairs: the leader's, for both CTAs' bytes)
      ptx::mbar_init(ptx::smem_u32(&c.full[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&c.empty[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&c.afull[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&c.aempty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(ptx::smem_u32(&c.tfull[a]), 1);
      ptx::mbar_init(ptx::smem_u32(&c.tempty[a]), EPI_WARPS * CG);   // one arrival per epilogue warp
    }
    ptx::mbar_init(ptx::smem_u32(&c.drain), 1);
    ptx::mbar_init(ptx::smem_u32(&c.never), 1);
    for (int q = 0; q < 4; ++q) {
      ptx::mbar_init(ptx::smem_u32(&c.xfull[q]), 32);
      ptx::mbar_init(ptx::smem_u32(&c.xempty[q]), 32);
    }
    c.abort = 0;
    ptx::fence_mbar_init();
    ptx::tma_prefetch(&tmA);
    ptx::tma_prefetch(&tmB0);
    ptx::tma_prefetch(&tmB1);
    if constexpr (MT::WGRAD) {
      ptx::tma_prefetch(&tmO0);
      ptx::tma_prefetch(&tmO1);
      if constexpr (!C::MX) {
        ptx::tma_prefetch(&tmAT);
        ptx::tma_prefetch(&tmBT);
      }
    }
  }
  if (warp == 1) {
    if constexpr (CG == 2) {
      ptx::tmem_alloc_pair(ptx::smem_u32(&c.tmem_base), C::TMEM_COLS);
      ptx::tmem_relinquish_pair();
    } else {
      ptx::tmem_alloc(ptx::smem_u32(&c.tmem_base), C::TMEM_COLS);
      ptx::tmem_relinquish();
    }
  }
  if constexpr (MODE == ROUTER) {
    if (warp >= 2 && warp < 2 + EPI_WARPS) {
      const float *bias = static_cast<const float *>(p.aux);
      for (int e = threadIdx.x - 64; e < MAX_E; e += 32 * EPI_WARPS) c.bias[e] = (bias && e < p.E) ? bias[e] : 0.f;
    }
  }
  // shared-memory copy of offsets: bf16 weight gradients in the control block's union (their
  // prefix is unused), row-grouped GEMMs after the control block; MXFP8 weight gradients read
  // the global array (their union holds the padded prefix)
  constexpr bool SMEM_OFFS = MODE != ROUTER && !(MT::WGRAD && C::MX);
  int *offs_smem = MT::WGRAD ? c.offs : reinterpret_cast<int *>(extra);
  const int *offs_s = SMEM_OFFS ? offs_smem : p.offsets;
  if constexpr (SMEM_OFFS) {
    if (warp == 3)
      for (int i = lane; i <= p.E; i += 32) offs_smem[i] = p.offsets[i];
    if (ASTAT && warp == 3) {
      // strips only when every expert's K-blocks fit the A slots: a strip of an expert that
      // streams A would hold its whole row of tiles on one CTA (pair) and stall the others
      __syncwarp();
      int mx = 0;
      for (int e = lane; e < p.E; e += 32) mx = max(mx, offs_smem[e + 1] - offs_smem[e]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) c.strips = p.strips && (mx + C::KBLK - 1) / C::KBLK <= p.na;
    }
  }
  if (warp == 2 && (!MT::WGRAD || C::MX) && MODE != ROUTER) {
    // per-expert 128-row block counts, exclusive prefix: lane l owns experts 8l..8l+7
    int cnt[8], s = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int e = lane * 8 + i;
      int n = 0;
      if (e < p.E) n = (p.offsets[e + 1] - p.offsets[e] + BMP - 1) / BMP;
      cnt[i] = n;
      s += n;
    }
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - s;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int e = lane * 8 + i;
      if (e < p.E) c.prefix[e] = run;
      run += cnt[i];
    }
    if (lane == 31) c.prefix[p.E] = incl;
  }
  ptx::tc_fence_before();
  __syncthreads();
  if constexpr (CG == 2) ptx::cluster_sync();   // the peer's barriers exist before anyone signals them
  ptx::tc_fence_after();
  const uint32_t tmem_base = c.tmem_base;
  const int ntiles = total_tiles<MODE, BN, CG>(p, c);
  // A stationary (bf16 weight gradients): the ring memory holds NA A slots and then SB B
  // slots instead of STAGES (A | B) stages.  With strips, CTA pairs (whose A and B slots are
  // the same size) split the ring's slots by the host's choice (p.na); otherwise, and for
  // single CTAs, STAGES of each.
  const bool strips = ASTAT && c.strips;
  const int NA = ASTAT ? ((C::A_BYTES == C::B_BYTES && strips) ? p.na : C::STAGES) : 0;
  const int SB = ASTAT ? 2 * C::STAGES - NA : C::STAGES;

  if (warp == 0) {
    // ================================================================ producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_par = 0;  // per stage: a fill is in flight / its parity
    uint32_t aph = 0, a_armed = 0, a_armed_par = 0;   // A slots: fill parity, in flight, its parity
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int t = nth_tile<BN>(i, p, tile0, tstep, ntiles, strips);
      if (t < 0) break;
      Tile tl;
      get_tile<MODE, BN, C::KBLK, C::MX, CG>(t, p, c, offs_s, tl, rank);
      // A stationary: the strip's first tile loads A (the K-blocks stay in their slots for
      // the strip's other tiles), unless there are more K-blocks than slots
      const bool a_res = strips && tl.num_kb <= NA;
      const bool load_a = ASTAT && (!a_res || i % (p.N / BN) == 0);
      for (int kb = 0; kb < tl.num_kb && ok; ++kb) {
        // bf16 weight gradients: the expert's last K-block, when partial, comes from the tail
        // buffers (rows e*64 + i: the block's rows, then zeros)
        bool tail = false;
        if constexpr (MT::WGRAD && !C::MX) tail = tl.rows - kb * C::KBLK < C::KBLK;
        if constexpr (ASTAT) {
          if (load_a) {
            const int as = a_res ? kb : kb % NA;
            if (lane == 0)
              ok = ptx::mbar_wait(ptx::smem_u32(&c.aempty[as]), ((aph >> as) & 1u) ^ 1u, abort_flag, WAIT_LIMIT_NS);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) { if (lane == 0) note_fail(p, 0, t, kb, 1); break; }
            if (lane == 0) {
              const uint32_t abar = ptx::smem_u32(&c.afull[as]);
              const uint32_t abar_leader = CG == 2 ? ptx::mapa(abar, 0) : abar;
              const uint32_t a_dst = ptx::smem_u32(ring + as * C::A_BYTES);
              if (rank == 0) ptx::mbar_arrive_expect_tx(abar, CG * C::A_BYTES);
#pragma unroll
              for (int j = 0; j < BM / C::BOX_MN; ++j) {
                const CUtensorMap *tm = tail ? &tmAT : &tmA;
                const int y = tail ? tl.e * C::KBLK : tl.row0 + kb * C::KBLK;
                if (CG == 2) ptx::tma_load_2d_pair(a_dst + j * C::BOX_BYTES, tm, abar_leader, tl.mcol0 + j * C::BOX_MN, y);
                else ptx::tma_load_2d(a_dst + j * C::BOX_BYTES, tm, abar, tl.mcol0 + j * C::BOX_MN, y);
              }
            }
            a_armed |= 1u << as;
            if ((aph >> as) & 1u) a_armed_par |= 1u << as; else a_armed_par &= ~(1u << as);
            aph ^= 1u << as;
          }
        }
        if (lane == 0) ok = ptx::mbar_wait(ptx::smem_u32(&c.empty[stage]), phase ^ 1, abort_flag, WAIT_LIMIT_NS);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { if (lane == 0) note_fail(p, 0, t, kb, 0); break; }
        const uint32_t a_dst = ptx::smem_u32(ring + stage * C::STAGE_BYTES);
        const uint32_t b_dst = ASTAT ? ptx::smem_u32(ring + NA * C::A_BYTES + stage * C::B_BYTES) : a_dst + C::A_BYTES;
        if (ASTAT) (void)a_dst;
        const uint32_t full_local = ptx::smem_u32(&c.full[stage]);
        // pairs: the bytes of both CTAs' loads are counted on the leader's full barrier
        const uint32_t full_leader = CG == 2 ? ptx::mapa(full_local, 0) : full_local;
        const uint32_t bar = full_local;
        auto ld = [&](uint32_t dst, const CUtensorMap *tm, int x, int y) {
          if (CG == 2) ptx::tma_load_2d_pair(dst, tm, full_leader, x, y);
          else ptx::tma_load_2d(dst, tm, bar, x, y);
        };
        if (lane == 0) {
          if (rank == 0) ptx::mbar_arrive_expect_tx(bar, ASTAT ? CG * C::B_BYTES : CG * C::STAGE_BYTES + C::SF_BYTES);
          if constexpr (C::MX) {
            // the stage's scale-factor tiles, A then B (512 bytes each), straight into the
            // arrangement the MMA issuer's tcgen05.cp reads
            int64_t a_mn, a_kg, b_mn, b_kg;
            if constexpr (MT::A_MN) { a_mn = tl.m_blk; a_kg = tl.row0 / 128 + kb; }
            else { a_mn = tl.row0 / 128; a_kg = kb; }
            if constexpr (MODE == FWD_GU || MODE == FWD_DOWN) {
              b_mn = (int64_t)tl.n_blk * BN / 128; b_kg = (int64_t)tl.e * p.K / 128 + kb;
            } else if constexpr (MODE == DGRAD_DOWN) {
              b_mn = ((int64_t)tl.e * p.f + (int64_t)tl.n_blk * BN) / 128; b_kg = kb;
            } else if constexpr (MODE == DGRAD_GU) {
              b_mn = ((int64_t)tl.e * p.d + (int64_t)tl.n_blk * BN) / 128; b_kg = kb;
            } else {
              b_mn = (int64_t)tl.n_blk * BN / 128; b_kg = tl.row0 / 128 + kb;
            }
            const uint32_t sf_dst = ptx::smem_u32(sf_ring + stage * C::SF_BYTES);
            ptx::bulk_load(sf_dst, p.sfa + (a_mn * p.nka + a_kg) * 512, 512, full_local);
            ptx::bulk_load(sf_dst + 512, p.sfb + (b_mn * p.nkb + b_kg) * 512, 512, full_local);
          }
          // ---- A (A stationary: loaded above, into its own slot)
          if constexpr (ASTAT) {
          } else if constexpr (MT::A_MN) {
#pragma unroll
            for (int i = 0; i < BM / C::BOX_MN; ++i) {
              if (tail) ld(a_dst + i * C::BOX_BYTES, &tmAT, tl.mcol0 + i * C::BOX_MN, tl.e * C::KBLK);
              else ld(a_dst + i * C::BOX_BYTES, &tmA, tl.mcol0 + i * C::BOX_MN, tl.row0 + kb * C::KBLK);
            }
          } else {
            ld(a_dst, &tmA, kb * C::KBLK, tl.row0);
          }
          // ---- B
          if constexpr (C::MX && MODE == FWD_GU) {
            // quantised [Wg | Wu] with gate and up interleaved in 64-column chunks
            ptx::tma_load_2d(b_dst, &tmB0, bar, tl.n_blk * BN, tl.e * p.K + kb * C::KBLK);
          } else if constexpr (C::MX && MODE == DGRAD_GU) {
            // quantised [Wg | Wu] rows (K = 2f), one tensor
            ptx::tma_load_2d(b_dst, &tmB0, bar, kb * C::KBLK, tl.e * p.d + tl.n_blk * BN);
          } else if constexpr (FWD_B_KMAJOR && MODE == FWD_GU) {
            // Wg^T, Wu^T [E*f][d]: gate rows then up rows of the 256-row B tile
            const int half = BN / 2;
            ptx::tma_load_2d(b_dst, &tmB0, bar, kb * C::KBLK, tl.e * p.f + tl.n_blk * half);
            ptx::tma_load_2d(b_dst + half * 128, &tmB1, bar, kb * C::KBLK, tl.e * p.f + tl.n_blk * half);
          } else if constexpr (FWD_B_KMAJOR && MODE == FWD_DOWN) {
            // Wd^T [E*d][f]
            ptx::tma_load_2d(b_dst, &tmB0, bar, kb * C::KBLK, tl.e * p.d + tl.n_blk * BN);
          } else if constexpr (MODE == FWD_GU && CG == 2) {
            // pair: the leader holds the gate half of B, the peer the up half
            const int half = BN / 2;
#pragma unroll
            for (int i = 0; i < half / C::BOX_MN; ++i)
              ld(b_dst + i * C::BOX_BYTES, rank == 0 ? &tmB0 : &tmB1, tl.n_blk * half + i * C::BOX_MN,
                 tl.e * p.K + kb * C::KBLK);
          } else if constexpr (MODE == FWD_GU) {
            const int half = BN / 2;
#pragma unroll
            for (int i = 0; i < half / C::BOX_MN; ++i) {
              ptx::tma_load_2d(b_dst + i * C::BOX_BYTES, &tmB0, bar, tl.n_blk * half + i * C::BOX_MN,
                               tl.e * p.K + kb * C::KBLK);
              ptx::tma_load_2d(b_dst + (half / C::BOX_MN + i) * C::BOX_BYTES, &tmB1, bar,
                               tl.n_blk * half + i * C::BOX_MN, tl.e * p.K + kb * C::KBLK);
            }
          } else if constexpr (MODE == ROUTER) {
            // W_r [d][E], MN-major; columns past E read as zeros
#pragma unroll
            for (int i = 0; i < BN / C::BOX_MN; ++i)
              ptx::tma_load_2d(b_dst + i * C::BOX_BYTES, &tmB0, bar, i * C::BOX_MN, kb * C::KBLK);
          } else if constexpr (MODE == FWD_DOWN) {
#pragma unroll
            for (int i = 0; i < BNC / C::BOX_MN; ++i)
              ld(b_dst + i * C::BOX_BYTES, &tmB0, tl.n_blk * BN + rank * BNC + i * C::BOX_MN,
                 tl.e * p.K + kb * C::KBLK);
          } else if constexpr (MODE == DGRAD_DOWN) {
            ld(b_dst, &tmB0, kb * C::KBLK, tl.e * p.f + tl.n_blk * BN + rank * BNC);
          } else if constexpr (MODE == DGRAD_GU) {
            const int kb_half = p.f / C::KBLK;
            if (kb < kb_half)
              ld(b_dst, &tmB0, kb * C::KBLK, tl.e * p.d + tl.n_blk * BN + rank * BNC);
            else
              ld(b_dst, &tmB1, (kb - kb_half) * C::KBLK, tl.e * p.d + tl.n_blk * BN + rank * BNC);
          } else {  // weight gradients: B is the MN-major activation gradient
#pragma unroll
            for (int i = 0; i < BNC / C::BOX_MN; ++i) {
              const int x = tl.n_blk * BN + rank * BNC + i * C::BOX_MN;
              if (tail) ld(b_dst + i * C::BOX_BYTES, &tmBT, x, tl.e * C::KBLK);
              else ld(b_dst + i * C::BOX_BYTES, &tmB0, x, tl.row0 + kb * C::KBLK);
            }
          }
        }
        // this stage's full barrier completes (or has completed) the phase of this pass
        armed |= 1u << stage;
        if (phase) armed_par |= 1u << stage; else armed_par &= ~(1u << stage);
        if (++stage == SB) { stage = 0; phase ^= 1; }
      }
    }
    // Drain: every TMA fill this warp issued must land before the CTA may exit, also after
    // an abort (these waits ignore the abort flag and give up only at the limit).  The last
    // fill of each stage is counted on its full barrier; earlier fills of a stage had landed
    // before the stage was refilled.  (Pairs: the leader's full barriers count the peer's
    // bytes too.)
    if (lane == 0) {
      for (int s = 0; s < 8; ++s) {
        if (rank == 0 && ((armed >> s) & 1u))
          if (!ptx::mbar_wait(ptx::smem_u32(&c.full[s]), (armed_par >> s) & 1u, nullptr, WAIT_LIMIT_NS))
            note_fail(p, 0, 0, s, 2);
        if (rank == 0 && ((a_armed >> s) & 1u))
          if (!ptx::mbar_wait(ptx::smem_u32(&c.afull[s]), (a_armed_par >> s) & 1u, nullptr, WAIT_LIMIT_NS))
            note_fail(p, 0, 0, s, 2);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = (1u << 4) | (ElemTraits<T>::FMT << 7) | (ElemTraits<T>::FMT << 10) |
                                 ((MT::A_MN ? 1u : 0u) << 15) | ((B_MN ? 1u : 0u) << 16) |
                                 ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BMP >> 4) << 24);
      // block-scaled E4M3 x E4M3 (formats 0), UE8M0 scales (bit 23); per-MMA scale-byte ids
      // go in bits 5:4 (B) and 30:29 (A)
      constexpr uint32_t idesc_mx = ((MT::A_MN ? 1u : 0u) << 15) | ((B_MN ? 1u : 0u) << 16) |
                                    ((uint32_t)(BN >> 3) << 17) | (1u << 23) | ((uint32_t)(BM >> 4) << 24);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      if (CG == 1 && p.stall_ns) {
        // failure-detection hook: a wait that nothing ends runs out, and every role aborts
        ok = ptx::mbar_wait(ptx::smem_u32(&c.never), 0, abort_flag, p.stall_ns);
        if (!ok) note_fail(p, 1, 0, 0, 3);
      }
      uint32_t a_ph = 0;   // A stationary: per A slot, the parity of its next fill
      for (;; ++it) {
        const int t = nth_tile<BN>(it, p, tile0, tstep, ntiles, strips);
        if (t < 0 || !ok) break;
        Tile tl;
        get_tile<MODE, BN, C::KBLK, C::MX, CG>(t, p, c, offs_s, tl, rank);
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        // A stationary: the strip's first tile waits for A, its last releases A's slots (every
        // tile, when A streams)
        const int nt_strip = ASTAT ? p.N / BN : 1;
        const bool a_res = strips && tl.num_kb <= NA;
        const bool wait_a = ASTAT && (!a_res || it % nt_strip == 0);
        const bool release_a = ASTAT && (!a_res || it % nt_strip == nt_strip - 1);
        ok = ptx::mbar_wait(ptx::smem_u32(&c.tempty[acc]), aph ^ 1, abort_flag, WAIT_LIMIT_NS);
        if (!ok) { note_fail(p, 1, t, 0, 0); break; }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        if (tl.num_kb == 0) {
          ptx::mbar_arrive(ptx::smem_u32(&c.tfull[acc]));
          if constexpr (CG == 2) ptx::mbar_arrive_cluster(ptx::mapa(ptx::smem_u32(&c.tfull[acc]), 1));
          continue;
        }
        for (int kb = 0; kb < tl.num_kb; ++kb) {
          int as = 0;
          if constexpr (ASTAT) {
            as = a_res ? kb : kb % NA;
            if (wait_a) {
              ok = ptx::mbar_wait(ptx::smem_u32(&c.afull[as]), (a_ph >> as) & 1u, abort_flag, WAIT_LIMIT_NS);
              if (!ok) { note_fail(p, 1, t, kb, 1); break; }
              a_ph ^= 1u << as;
            }
          }
          // loaded bytes and commit arrivals are ordered by the barrier itself
          ok = ptx::mbar_wait(ptx::smem_u32(&c.full[stage]), phase, abort_flag, WAIT_LIMIT_NS);
          if (!ok) { note_fail(p, 1, t, kb, 1); break; }
          ptx::tc_fence_after();
          const uint32_t a_addr = ASTAT ? ptx::smem_u32(ring + as * C::A_BYTES)
                                        : ptx::smem_u32(ring + stage * C::STAGE_BYTES);
          const uint32_t b_addr = ASTAT ? ptx::smem_u32(ring + NA * C::A_BYTES + stage * C::B_BYTES)
                                        : a_addr + C::A_BYTES;
          uint32_t sfa_t = 0, sfb_t = 0;
          if constexpr (C::MX) {
            // scales of this stage into TMEM columns 2*BN (A) and 2*BN + 4 (B)
            sfa_t = tmem_base + 2 * BN;
            sfb_t = sfa_t + 4;
            const uint32_t sf_s = ptx::smem_u32(sf_ring + stage * C::SF_BYTES);
            ptx::tmem_cp_32x128b_x4(sfa_t, ptx::smem_desc_sf(sf_s));
            ptx::tmem_cp_32x128b_x4(sfb_t, ptx::smem_desc_sf(sf_s + 512));
          }
          // a weight-gradient tail stage: only the UMMA_K-row slices that hold expert rows (the
          // rest of the tail buffer's block is zeros)
          int nk = C::KBLK / C::UMMA_K;
          if constexpr (MT::WGRAD && !C::MX)
            nk = min(nk, (tl.rows - kb * C::KBLK + C::UMMA_K - 1) / C::UMMA_K);
#pragma unroll
          for (int kk = 0; kk < C::KBLK / C::UMMA_K; ++kk) {
            if (kk >= nk) break;
            uint64_t adesc, bdesc;
            if constexpr (MT::A_MN)
              adesc = ptx::smem_desc_sw128(a_addr + kk * C::UMMA_K * 128, C::BOX_BYTES, 1024);
            else
              adesc = ptx::smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            if constexpr (B_MN)
              bdesc = ptx::smem_desc_sw128(b_addr + kk * C::UMMA_K * 128, C::BOX_BYTES, 1024);
            else
              bdesc = ptx::smem_desc_sw128(b_addr + kk * 32, 16, 1024);
            const uint32_t accum = (kb | kk) ? 1u : 0u;
            if constexpr (C::MX)
              ptx::mma_mxf8(d_tmem, adesc, bdesc, idesc_mx | ((uint32_t)kk << 4) | ((uint32_t)kk << 29),
                            sfa_t | ((uint32_t)kk << 30), sfb_t | ((uint32_t)kk << 30), accum);
            else if constexpr (CG == 2) ptx::mma_f16_pair(d_tmem, adesc, bdesc, idesc, accum);
            else if constexpr (sizeof(T) == 2) ptx::mma_f16(d_tmem, adesc, bdesc, idesc, accum);
            else ptx::mma_tf32(d_tmem, adesc, bdesc, idesc, accum);
          }
          if constexpr (CG == 2) ptx::tc_commit_pair_mc(ptx::smem_u32(&c.empty[stage]), 0x3);
          else ptx::tc_commit(ptx::smem_u32(&c.empty[stage]));
          if (ASTAT && release_a) {
            if constexpr (CG == 2) ptx::tc_commit_pair_mc(ptx::smem_u32(&c.aempty[as]), 0x3);
            else ptx::tc_commit(ptx::smem_u32(&c.aempty[as]));
          }
          if (++stage == SB) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if constexpr (CG == 2) ptx::tc_commit_pair_mc(ptx::smem_u32(&c.tfull[acc]), 0x3);
        else ptx::tc_commit(ptx::smem_u32(&c.tfull[acc]));
      }
      // Drain: all MMAs issued here complete before TMEM is freed, also after an abort.
      if constexpr (CG == 2) ptx::tc_commit_pair(ptx::smem_u32(&c.drain));
      else ptx::tc_commit(ptx::smem_u32(&c.drain));
      if (!ptx::mbar_wait(ptx::smem_u32(&c.drain), 0, nullptr, WAIT_LIMIT_NS)) note_fail(p, 1, 0, 0, 2);
    }
    __syncwarp();
  } else {
    // ================================================================ epilogue
    using OutT = typename ElemTraits<T>::Out;
    // EPI_WARPS warps: warp w reads TMEM lane quarter w % 4 (one tile row per thread);
    // the two warps of a quarter split the accumulator's columns in halves.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;     // 0 or 1
    const int r = q * 32 + lane;          // tile row owned by this thread
    uint8_t *epi_box = extra + (warp - 2) * EPI_BOX_BYTES;       // weight gradients
    for (int it = 0;; ++it) {
      const int t = nth_tile<BN>(it, p, tile0, tstep, ntiles, strips);
      if (t < 0) break;
      Tile tl;
      get_tile<MODE, BN, C::KBLK, C::MX, CG>(t, p, c, offs_s, tl, rank);
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      bool ok = ptx::mbar_wait(ptx::smem_u32(&c.tfull[acc]), aph, abort_flag, WAIT_LIMIT_NS);
      if (!__all_sync(0xffffffffu, ok)) { if (lane == 0) note_fail(p, 2, t, 0, 0); break; }
      ptx::tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;

      if constexpr (MODE == ROUTER) {
        // One token per tile row.  The two warps of a lane quarter split the experts in
        // halves and each takes the k best of its half by k max passes over the order keys
        // (a pass keeps the first of equal keys, so ties go to the lower expert, and drops the
        // previous pass's pick); the first warp then merges the second warp's picks into its
        // own through shared memory and writes the gates, the softmax of the k logits.
        constexpr int HC = BN / 2;
        const int cb = half * HC;                         // first expert of this half
        const int ncol = min(HC, max(0, p.E - cb));
        const bool two = p.E > HC;                        // the second half holds experts
        const bool valid = r < tl.rows;
        const int64_t row = (int64_t)tl.orow0 + r;
        float *logits = static_cast<float *>(p.out2);
        bool nan_seen = false;
        uint32_t pk[MAX_K];
        int pe[MAX_K];
        if (ncol > 0) {
          auto load = [&](int cc, float (&v)[32]) {
            ptx::tmem_ld32(taddr + cb + cc, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] += c.bias[cb + cc + i];
          };
          auto put_logits = [&](int cc, const float (&v)[32]) {
            if (!valid || !logits) return;
            float *dst = logits + row * p.E + cb + cc;
            if (cb + cc + 32 <= p.E) {
              store32(dst, v);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (cb + cc + i < p.E) dst[i] = v[i];
            }
          };
          if constexpr (HC <= 64) {
            // keys of the whole half stay in registers
            uint32_t o[HC];
#pragma unroll
            for (int cc = 0; cc < HC; cc += 32) {
              if (cc < ncol) {
                float v[32];
                load(cc, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                  o[cc + i] = cc + i < ncol ? router_key(v[i]) : 0u;
                  nan_seen |= o[cc + i] == 1u;
                }
                put_logits(cc, v);
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) o[cc + i] = 0u;
              }
            }
            int prev = -1;
#pragma unroll
            for (int j = 0; j < MAX_K; ++j) {
              pk[j] = 0u;
              pe[j] = INT_MAX;
              if (j < p.k) {
                uint32_t bo[4] = {0u, 0u, 0u, 0u};
                int bi[4] = {0, 0, 0, 0};
#pragma unroll
                for (int i = 0; i < HC; ++i) {
                  if (i == prev) o[i] = 0u;
                  if (o[i] > bo[i & 3]) { bo[i & 3] = o[i]; bi[i & 3] = i; }
                }
                uint32_t best = bo[0];
                int bc = bi[0];
#pragma unroll
                for (int a = 1; a < 4; ++a)
                  if (key_above(bo[a], bi[a], best, bc)) { best = bo[a]; bc = bi[a]; }
                prev = best ? bc : -1;
                pk[j] = best;
                pe[j] = best ? cb + bc : INT_MAX;
              }
            }
          } else {
            // wide halves: every pass reads the accumulator again and keeps the best key
            // that ranks below the previous pick
#pragma unroll 1
            for (int cc = 0; cc < ncol; cc += 32) {
              float v[32];
              load(cc, v);
#pragma unroll
              for (int i = 0; i < 32; ++i) nan_seen |= (cc + i < ncol) && (v[i] != v[i]);
              put_logits(cc, v);
            }
            uint32_t po = 0xffffffffu;
            int pc = -1;
#pragma unroll
            for (int j = 0; j < MAX_K; ++j) {
              pk[j] = 0u;
              pe[j] = INT_MAX;
              if (j < p.k) {
                uint32_t bo[4] = {0u, 0u, 0u, 0u};
                int bi[4] = {0, 0, 0, 0};
#pragma unroll 1
                for (int cc = 0; cc < ncol; cc += 32) {
                  float v[32];
                  load(cc, v);
#pragma unroll
                  for (int i = 0; i < 32; ++i) {
                    const int col = cc + i;
                    uint32_t o = col < ncol ? router_key(v[i]) : 0u;
                    if (!(o < po || (o == po && col > pc))) o = 0u;
                    if (o > bo[i & 3]) { bo[i & 3] = o; bi[i & 3] = col; }
                  }
                }
                uint32_t best = bo[0];
                int bc = bi[0];
#pragma unroll
                for (int a = 1; a < 4; ++a)
                  if (key_above(bo[a], bi[a], best, bc)) { best = bo[a]; bc = bi[a]; }
                po = best ? best : 0u;
                pc = best ? bc : HC;
                pk[j] = best;
                pe[j] = best ? cb + bc : INT_MAX;
              }
            }
          }
        }
        if (valid && nan_seen) set_error(p.err, MOE_ERR_DEVICE_NAN);
        if (two) {
          uint32_t *xk = xbuf;
          int *xe = reinterpret_cast<int *>(xbuf + MAX_K * BM);
          if (half == 1) {
            if (it > 0) ok = ptx::mbar_wait(ptx::smem_u32(&c.xempty[q]), (it - 1) & 1, abort_flag, WAIT_LIMIT_NS);
            if (ok) {
#pragma unroll
              for (int j = 0; j < MAX_K; ++j)
                if (j < p.k) { xk[j * BM + r] = pk[j]; xe[j * BM + r] = pe[j]; }
              ptx::mbar_arrive(ptx::smem_u32(&c.xfull[q]));
            }
          } else {
            ok = ptx::mbar_wait(ptx::smem_u32(&c.xfull[q]), it & 1, abort_flag, WAIT_LIMIT_NS);
            if (ok) {
#pragma unroll
              for (int m = 0; m < MAX_K; ++m) {
                if (m < p.k) {
                  uint32_t xo = xk[m * BM + r];
                  int xi = xe[m * BM + r];
#pragma unroll
                  for (int j = 0; j < MAX_K; ++j) {
                    if (j < p.k && key_above(xo, xi, pk[j], pe[j])) {
                      const uint32_t so = pk[j];
                      const int si = pe[j];
                      pk[j] = xo; pe[j] = xi; xo = so; xi = si;
                    }
                  }
                }
              }
              ptx::mbar_arrive(ptx::smem_u32(&c.xempty[q]));
            }
          }
          if (!__all_sync(0xffffffffu, ok)) { if (lane == 0) note_fail(p, 2, t, 0, 3); break; }
        }
        if (half == 0 && valid) {
          int32_t *idx = static_cast<int32_t *>(p.out0);
          float *gate = static_cast<float *>(p.out1);
          float ex[MAX_K], sum = 0.f;
          const float z0 = router_key_value(pk[0]);
#pragma unroll
          for (int j = 0; j < MAX_K; ++j) {
            ex[j] = 0.f;
            if (j < p.k) { ex[j] = expf(router_key_value(pk[j]) - z0); sum += ex[j]; }
          }
          const float inv = 1.0f / sum;
#pragma unroll
          for (int j = 0; j < MAX_K; ++j)
            if (j < p.k) { idx[row * p.k + j] = pe[j]; gate[row * p.k + j] = ex[j] * inv; }
        }
      } else if constexpr (MODE == FWD_GU) {
        // columns [0, BN/2) hold h = x Wg, [BN/2, BN) hold u = x Wu for the same f-range;
        // either output may be absent (h, u not kept when the backward recomputes them; a not
        // needed when the backward recomputes h, u)
        const bool valid = r < tl.rows;
        const int nvalid = min(32, max(0, tl.rows - q * 32));
        const int64_t srow = (int64_t)tl.orow0 + q * 32;      // output row of slab row 0
        OutT *hu = static_cast<OutT *>(p.out0);
        OutT *aa = static_cast<OutT *>(p.out1);
#pragma unroll 1
        for (int cc = half * (BN / 4); cc < (half + 1) * (BN / 4); cc += 32) {
          float h[32], u[32];
          ptx::tmem_ld32(taddr + cc, h);
          ptx::tmem_ld32(taddr + BN / 2 + cc, u);
          const int col = tl.n_blk * (BN / 2) + cc;
          if (hu) {
            store_slab(hu + srow * 2 * p.f + col, 2 * p.f, nvalid, h);
            store_slab(hu + srow * 2 * p.f + p.f + col, 2 * p.f, nvalid, u);
          }
          if (aa) {
            float a[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) a[i] = valid ? h[i] * sigmoidf_(h[i]) * u[i] : 0.f;
            store_slab(aa + srow * p.f + col, p.f, nvalid, a);
            if constexpr (C::MX) {
              if (p.q_row_codes) {
                // the down projection's operand: the stored bf16 a, in MXFP8 along f, at the
                // padded row (pad rows hold zeros)
                const int64_t prow = (int64_t)tl.row0 + r;
#pragma unroll
                for (int i = 0; i < 32; ++i) a[i] = __bfloat162float(__float2bfloat16_rn(a[i]));
                mx_block32_store(a, p.q_row_codes + prow * p.f + col,
                                 p.q_row_scales + sf_tiled_off(prow, col / 32, p.nk_row));
                if (p.q_col_codes)   // and down the padded token axis (the weight gradient's operand)
                  mx_slab32_cols_store(a, p.q_col_codes + prow * p.f + col,
                                       p.q_col_scales + sf_tiled_off(col + lane, prow / 32, p.nk_col));
              }
            }
          }
        }
      } else if constexpr (MODE == FWD_DOWN || MODE == DGRAD_GU) {
        const int nvalid = min(32, max(0, tl.rows - q * 32));
        const int64_t srow = (int64_t)tl.orow0 + q * 32;
        OutT *out = static_cast<OutT *>(p.out0);
#pragma unroll 1
        for (int cc = half * (BN / 2); cc < (half + 1) * (BN / 2); cc += 32) {
          float v[32];
          ptx::tmem_ld32(taddr + cc, v);
          store_slab(out + srow * p.N + tl.n_blk * BN + cc, p.N, nvalid, v);
        }
      } else if constexpr (MODE == DGRAD_DOWN) {
        // da -> (dh, du) through the SwiGLU derivative, using the saved h and u.  The
        // loads of the next chunk's h, u are issued before this chunk's math.
        const bool valid = r < tl.rows;
        const int nvalid = min(32, max(0, tl.rows - q * 32));
        const int64_t row = (int64_t)tl.orow0 + r;
        const int64_t srow = (int64_t)tl.orow0 + q * 32;
        const OutT *hu = static_cast<const OutT *>(p.aux);
        OutT *dhu = static_cast<OutT *>(p.out0);
        constexpr int NV = 32 / Vec<OutT>::N;   // 16-byte vectors per 32 values
        constexpr int VN = Vec<OutT>::N;
        const int c0 = half * (BN / 2), c1 = (half + 1) * (BN / 2);
        uint4 hv[2][NV], uv[2][NV];
        auto issue = [&](int buf, int cc) {
          const uint4 *hs = reinterpret_cast<const uint4 *>(hu + row * 2 * p.f + tl.n_blk * BN + cc);
          const uint4 *us = reinterpret_cast<const uint4 *>(hu + row * 2 * p.f + p.f + tl.n_blk * BN + cc);
#pragma unroll
          for (int i = 0; i < NV; ++i) {
            hv[buf][i] = valid ? __ldg(hs + i) : make_uint4(0, 0, 0, 0);
            uv[buf][i] = valid ? __ldg(us + i) : make_uint4(0, 0, 0, 0);
          }
        };
        issue(0, c0);
#pragma unroll
        for (int j = 0; j < (BN / 2) / 32; ++j) {
          const int cc = c0 + j * 32;
          float da[32];
          ptx::tmem_ld32(taddr + cc, da);
          if (cc + 32 < c1) issue((j + 1) & 1, cc + 32);
          float dh[32], du[32];
#pragma unroll
          for (int i = 0; i < NV; ++i) {   // one 16-byte vector of h, u at a time
            float h[VN], u[VN];
            Vec<OutT>::load(hv[j & 1][i], h);
            Vec<OutT>::load(uv[j & 1][i], u);
#pragma unroll
            for (int v = 0; v < VN; ++v) {
              const float g = da[i * VN + v];
              const float s = sigmoidf_(h[v]);
              dh[i * VN + v] = g * u[v] * s * (1.0f + h[v] * (1.0f - s));
              du[i * VN + v] = g * h[v] * s;
            }
          }
          const int col = tl.n_blk * BN + cc;
          if (dhu) {   // (the MXFP8 layer keeps [dh | du] in MXFP8 only)
            store_slab(dhu + srow * 2 * p.f + col, 2 * p.f, nvalid, dh);
            store_slab(dhu + srow * 2 * p.f + p.f + col, 2 * p.f, nvalid, du);
          }
          if constexpr (C::MX) {
            if (p.q_row_codes) {
              // the gate/up GEMMs' operand: the stored bf16 [dh | du] in MXFP8 along 2f (for the
              // data gradient) and down the padded token axis (for the weight gradient); pad
              // rows hold zeros
              const int64_t prow = (int64_t)tl.row0 + r;
              const int64_t ld = 2 * p.f;
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                dh[i] = valid ? __bfloat162float(__float2bfloat16_rn(dh[i])) : 0.f;
                du[i] = valid ? __bfloat162float(__float2bfloat16_rn(du[i])) : 0.f;
              }
              mx_block32_store(dh, p.q_row_codes + prow * ld + col,
                               p.q_row_scales + sf_tiled_off(prow, col / 32, p.nk_row));
              mx_block32_store(du, p.q_row_codes + prow * ld + p.f + col,
                               p.q_row_scales + sf_tiled_off(prow, (p.f + col) / 32, p.nk_row));
              const int64_t kb = prow / 32;   // every lane of the warp: the same 32-row block
              mx_slab32_cols_store(dh, p.q_col_codes + prow * ld + col,
                                   p.q_col_scales + sf_tiled_off(col + lane, kb, p.nk_col));
              mx_slab32_cols_store(du, p.q_col_codes + prow * ld + p.f + col,
                                   p.q_col_scales + sf_tiled_off(p.f + col + lane, kb, p.nk_col));
            }
          }
        }
      } else {  // weight gradients: rows q*32.. of the [M x N] block of expert e
        // The warp's 32 x 128 part of the accumulator is read and rounded to bf16 first and
        // the accumulator released, so that the MMAs of the tile after next need not wait for
        // the stores.  Each 32 x 64 piece then goes through the warp's staging box in the
        // layout of a 128-byte-swizzled TMA box (16-byte chunk j of row r at chunk j ^ (r % 8));
        // one lane stores the box with TMA.  The box is refilled only once the store that last
        // used it has read it.
        static_assert(sizeof(OutT) == 2, "weight gradients are stored as bf16");
        constexpr int PIECES = BN / 2 / 64;
        uint4 pk[PIECES][8];
#pragma unroll
        for (int pc = 0; pc < PIECES; ++pc) {
          float v0[32], v1[32];
          const int cc = half * (BN / 2) + pc * 64;
          if (tl.num_kb > 0) {
            ptx::tmem_ld32(taddr + cc, v0);
            ptx::tmem_ld32(taddr + cc + 32, v1);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) { v0[i] = 0.f; v1[i] = 0.f; }
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) pk[pc][j] = Vec<OutT>::store(j < 4 ? &v0[8 * j] : &v1[8 * (j - 4)]);
        }
        // release the accumulator: one arrival per warp on the leader's barrier
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (CG == 2 && rank != 0) ptx::mbar_arrive_cluster(ptx::mapa(ptx::smem_u32(&c.tempty[acc]), 0));
          else ptx::mbar_arrive(ptx::smem_u32(&c.tempty[acc]));
        }
        const int orow = tl.e * p.M + tl.mcol0 + q * 32;
#pragma unroll
        for (int pc = 0; pc < PIECES; ++pc) {
          const int cc = half * (BN / 2) + pc * 64;
          uint8_t *box = epi_box;
          if (lane == 0) ptx::bulk_wait_read<0>();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4 *>(box + lane * 128 + ((j ^ (lane & 7)) << 4)) = pk[pc][j];
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int col = tl.n_blk * BN + cc;
            if constexpr (MODE == WGRAD_DOWN) {
              ptx::tma_store_2d(&tmO0, ptx::smem_u32(box), col, orow);
            } else {
              // N runs over [dh | du]: columns below f are dW_gate, the rest dW_up
              if (col < p.f) ptx::tma_store_2d(&tmO0, ptx::smem_u32(box), col, orow);
              else ptx::tma_store_2d(&tmO1, ptx::smem_u32(box), col - p.f, orow);
            }
            ptx::bulk_commit();
          }
        }
      }
      if constexpr (!MT::WGRAD) {
        // release the accumulator: one arrival per warp on the leader's barrier
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (CG == 2 && rank != 0) ptx::mbar_arrive_cluster(ptx::mapa(ptx::smem_u32(&c.tempty[acc]), 0));
          else ptx::mbar_arrive(ptx::smem_u32(&c.tempty[acc]));
        }
      }
    }
    // weight gradients: the staging boxes stay in use until their TMA stores complete
    if constexpr (MT::WGRAD)
      if (lane == 0) ptx::bulk_wait_all();
  }

  // ------------------------------------------------------------------ teardown
  ptx::tc_fence_before();
  __syncthreads();
  // pairs: the leader's MMAs read the peer's shared memory and write its TMEM; neither CTA
  // leaves or frees TMEM before both are done (every wait above is bounded, so both get here)
  if constexpr (CG == 2) ptx::cluster_sync();
  if (threadIdx.x == 0 && c.abort) set_error(p.err, MOE_ERR_DEVICE_TIMEOUT);
  if (warp == 1) {
    ptx::tc_fence_after();
    if constexpr (CG == 2) ptx::tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else ptx::tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side
// A process may drive several GPUs, from several host threads: facts about a device are
// cached per device ordinal (0 = not known yet), and the driver entry point once.
constexpr int MAX_DEVICES = 64;

static int device_ordinal() {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < MAX_DEVICES ? dev : -1;
}

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}

// 2D row-major tensor [rows][cols], box [box_rows][box_cols], 128-byte swizzle.
static bool make_tmap(CUtensorMap *m, const void *ptr, int es, uint64_t cols, uint64_t rows,
                      uint32_t box_cols, uint32_t box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t gdim[2] = {cols, rows};
  cuuint64_t gstride[1] = {cols * (uint64_t)es};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estride[2] = {1, 1};
  const CUtensorMapDataType dt = es == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUresult r = enc(m, dt, 2,
                   const_cast<void *>(ptr), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace gg

int device_sm_count() {
  static std::atomic<int> cache[gg::MAX_DEVICES];
  const int dev = gg::device_ordinal();
  if (dev >= 0) {
    const int n = cache[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
  }
  int n = 0;
  if (dev < 0 || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev >= 0) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

namespace gg {
static int sm_count() { return device_sm_count(); }

// Failure-detection test hook (moe_debug_set_gemm_stall_ns), 0 in normal use: process-wide,
// read at each launch, applied to single-CTA launches only.
static std::atomic<uint64_t> g_stall_ns{0};

// Persistent launch: one CTA per SM (CG = 1), or one CTA pair per two SMs in clusters
// of two (CG = 2); never more CTAs (pairs) than tiles.
template <typename T, int BN, int MODE, int CG = 1>
static int launch(const CUtensorMap &a, const CUtensorMap &b0, const CUtensorMap &b1, const Params &p_in,
                  int64_t max_tiles, cudaStream_t st, const CUtensorMap *o0 = nullptr,
                  const CUtensorMap *o1 = nullptr, const CUtensorMap *at = nullptr,
                  const CUtensorMap *bt = nullptr) {
  using C = Cfg<T, BN, CG, extra_smem<MODE>()>;
  Params p = p_in;
  p.stall_ns = CG == 1 ? g_stall_ns.load(std::memory_order_relaxed) : 0;
  auto kern = grouped_gemm_kernel<T, BN, MODE, CG>;
  constexpr int SMEM = C::SMEM_BYTES;
  static_assert(SMEM <= SMEM_LIMIT, "shared memory");
  if (ModeTraits<MODE>::WGRAD && (!o0 || !o1)) return MOE_ERR_INVALID_ARG;
  if (ModeTraits<MODE>::WGRAD && !C::MX && (!at || !bt)) return MOE_ERR_INVALID_ARG;
  const CUtensorMap &out0 = o0 ? *o0 : a, &out1 = o1 ? *o1 : a;
  const CUtensorMap &atail = at ? *at : a, &btail = bt ? *bt : a;
  // bf16 weight gradients: A slots for 1.5x the average expert's K-blocks (4..8 of the 12
  // slots of a pair's ring), and whole strips per CTA (pair) when the average expert's A fits
  // and there are at least two strips per CTA (pair) to balance the load; otherwise A streams
  // tile by tile through half of the slots
  auto set_astat = [&](int64_t units) {
    if constexpr (ModeTraits<MODE>::WGRAD && !C::MX) {
      const int64_t avg_rows = p.E > 0 ? (int64_t)p.P / p.E : 0;
      const int64_t avg_kb = (avg_rows + C::KBLK - 1) / C::KBLK;
      if constexpr (C::A_BYTES == C::B_BYTES)
        p.na = (int)std::min<int64_t>(std::max<int64_t>((3 * avg_rows + 2 * C::KBLK - 1) / (2 * C::KBLK), 4), 8);
      else
        p.na = C::STAGES;
      const int64_t nstrips = (int64_t)p.E * (p.M / C::BMP);
      p.strips = avg_kb <= p.na && nstrips >= 2 * units;
      if (!p.strips) p.na = C::STAGES;   // A streams with B: as many slots of each
    }
  };
  // the shared-memory opt-in is a per-device property of the kernel: set once per device
  // (two threads racing here both set it, which is harmless)
  static std::atomic<bool> attr_set[MAX_DEVICES];
  const int dev = device_ordinal();
  if (dev < 0 || !attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (dev >= 0) attr_set[dev].store(true, std::memory_order_release);
  }
  if constexpr (CG == 1) {
    const int64_t units = std::min<int64_t>(sm_count(), std::max<int64_t>(max_tiles, 1));
    set_astat(units);
    kern<<<(unsigned)units, NUM_THREADS, SMEM, st>>>(a, b0, b1, out0, out1, atail, btail, p);
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CG;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // A persistent grid must be fully resident: pairs of SMs are taken inside one GPC, so
    // fewer than sm_count/2 pairs may fit at once (a late pair would run after a whole
    // persistent pair has finished).  Ask the occupancy calculator, once per device.
    static std::atomic<int> pairs_cache[MAX_DEVICES];
    int max_pairs = dev >= 0 ? pairs_cache[dev].load(std::memory_order_relaxed) : 0;
    if (max_pairs <= 0) {
      cfg.gridDim = dim3((unsigned)(sm_count() / CG * CG));
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) n = sm_count() / CG;
      max_pairs = std::min(n, sm_count() / CG);
      if (dev >= 0) pairs_cache[dev].store(max_pairs, std::memory_order_relaxed);
    }
    const int64_t units = std::min<int64_t>(max_pairs, std::max<int64_t>(max_tiles, 1));
    set_astat(units);
    cfg.gridDim = dim3((unsigned)(units * CG));
    if (cudaLaunchKernelEx(&cfg, kern, a, b0, b1, out0, out1, atail, btail, p) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Row-grouped GEMMs use 256-row CTA-pair tiles only when experts hold many rows: the
// last tile of each expert is on average half empty, which small groups cannot afford.
#ifndef MOE_PAIR_MIN_ROWS_PER_EXPERT
#define MOE_PAIR_MIN_ROWS_PER_EXPERT 768
#endif
static bool pair_rows(const Shape &s) { return s.P() >= MOE_PAIR_MIN_ROWS_PER_EXPERT * (int64_t)s.E; }

template <typename T>
static int fwd_impl(const Shape &s, const void *x_perm, const int32_t *offsets, const void *w_gate,
                    const void *w_up, const void *w_down, void *hu, void *a, void *y_perm, void *ws,
                    cudaStream_t st) {
  int *err = err_word(ws);
  if constexpr (sizeof(T) == 4) {
    // tf32 MMAs take K-major operands only: stage Wg^T, Wu^T [E][f][d] and Wd^T [E][d][f]
    WsLayout L = ws_layout(s);
    char *w = static_cast<char *>(ws);
    float *wgt = reinterpret_cast<float *>(w + L.wt), *wut = wgt + (size_t)s.E * s.d * s.f,
          *wdt = wut + (size_t)s.E * s.d * s.f;
    if (launch_transpose_batched(static_cast<const float *>(w_gate), wgt, s.E, s.d, s.f, st) ||
        launch_transpose_batched(static_cast<const float *>(w_up), wut, s.E, s.d, s.f, st) ||
        launch_transpose_batched(static_cast<const float *>(w_down), wdt, s.E, s.f, s.d, st))
      return MOE_ERR_CUDA;
    w_gate = wgt; w_up = wut; w_down = wdt;
  }
  constexpr int ES = sizeof(T);
  constexpr int KBLK = 128 / ES, BOX_MN = 128 / ES;
  const int64_t P = s.P();
  CUtensorMap tA, tB0, tB1;
  Params p{};
  p.offsets = offsets; p.E = s.E; p.P = (int)P; p.f = s.f; p.d = s.d; p.err = err; p.where = err + 1;
  const int64_t mblocks = (P + BM - 1) / BM + s.E;
  // GEMM 1: [h | u] = x_perm [P,d] x [Wg | Wu] [d,f]; N tile = 128 gate + 128 up columns
  {
    constexpr int BN = 256;
    if (!make_tmap(&tA, x_perm, ES, s.d, P, KBLK, BM)) return MOE_ERR_CUDA;
    if constexpr (sizeof(T) == 4) {
      if (!make_tmap(&tB0, w_gate, ES, s.d, (uint64_t)s.E * s.f, KBLK, BN / 2)) return MOE_ERR_CUDA;
      if (!make_tmap(&tB1, w_up, ES, s.d, (uint64_t)s.E * s.f, KBLK, BN / 2)) return MOE_ERR_CUDA;
    } else {
      if (!make_tmap(&tB0, w_gate, ES, s.f, (uint64_t)s.E * s.d, BOX_MN, KBLK)) return MOE_ERR_CUDA;
      if (!make_tmap(&tB1, w_up, ES, s.f, (uint64_t)s.E * s.d, BOX_MN, KBLK)) return MOE_ERR_CUDA;
    }
    p.K = s.d; p.N = 2 * s.f; p.out0 = hu; p.out1 = a; p.aux = nullptr;
    int rc = -1;
    if constexpr (sizeof(T) == 2)
      if (pair_rows(s)) rc = launch<T, BN, FWD_GU, 2>(tA, tB0, tB1, p, ((P + 255) / 256 + s.E) * (p.N / BN), st);
    if (rc < 0) rc = launch<T, BN, FWD_GU>(tA, tB0, tB1, p, mblocks * (p.N / BN), st);
    if (rc) return rc;
  }
  if (!y_perm) return MOE_OK;   // [h | u] only (the backward's recompute)
  // GEMM 2: y_perm = a [P,f] x Wd [f,d]
  {
    if (!make_tmap(&tA, a, ES, s.f, P, KBLK, BM)) return MOE_ERR_CUDA;
    p.K = s.f; p.N = s.d; p.out0 = y_perm; p.out1 = nullptr;
    int rc;
    const int bn = (s.d % 256 == 0) ? 256 : 128;
    bool ok;
    if constexpr (sizeof(T) == 4)
      ok = make_tmap(&tB0, w_down, ES, s.f, (uint64_t)s.E * s.d, KBLK, bn);
    else
      ok = make_tmap(&tB0, w_down, ES, s.d, (uint64_t)s.E * s.f, BOX_MN, KBLK);
    if (!ok) return MOE_ERR_CUDA;
    rc = -1;
    if constexpr (sizeof(T) == 2)
      if (bn == 256 && pair_rows(s))
        rc = launch<T, 256, FWD_DOWN, 2>(tA, tB0, tB0, p, ((P + 255) / 256 + s.E) * (p.N / 256), st);
    if (rc >= 0) {
    } else if (bn == 256)
      rc = launch<T, 256, FWD_DOWN>(tA, tB0, tB0, p, mblocks * (p.N / 256), st);
    else
      rc = launch<T, 128, FWD_DOWN>(tA, tB0, tB0, p, mblocks * (p.N / 128), st);
    if (rc) return rc;
  }
  return MOE_OK;
}

template <typename T>
static int bwd_impl(const Shape &s, const void *dy_perm, const void *x_perm, const void *hu,
                    const void *a, const int32_t *offsets, const void *w_gate, const void *w_up,
                    const void *w_down, void *dhu, void *dx_perm, void *dw_gate, void *dw_up,
                    void *dw_down, void *ws, cudaStream_t st) {
  constexpr int ES = sizeof(T);
  constexpr int KBLK = 128 / ES, BOX_MN = 128 / ES;
  static_assert(KBLK == WGRAD_TAIL_ROWS, "tail buffers hold one K-block per expert");
  const int64_t P = s.P();
  int *err = err_word(ws);
  const WsLayout L = ws_layout(s);
  void *tail_a = static_cast<char *>(ws) + L.wg_tail_a, *tail_b = static_cast<char *>(ws) + L.wg_tail_b;
  const uint64_t tail_rows = (uint64_t)s.E * WGRAD_TAIL_ROWS;
  CUtensorMap tA, tB0, tB1, tAT, tBT;
  Params p{};
  p.offsets = offsets; p.E = s.E; p.P = (int)P; p.f = s.f; p.d = s.d; p.err = err; p.where = err + 1;
  const int64_t mblocks = (P + BM - 1) / BM + s.E;
  int rc;
  // (1) da = dy_perm [P,d] x Wd^T [d,f]  -> SwiGLU backward -> dhu [P,2f]
  {
    if (!make_tmap(&tA, dy_perm, ES, s.d, P, KBLK, BM)) return MOE_ERR_CUDA;
    p.K = s.d; p.N = s.f; p.out0 = dhu; p.aux = hu;
    const int64_t pblocks = (P + 255) / 256 + s.E;
    if (s.f % 256 == 0 && pair_rows(s)) {
      if (!make_tmap(&tB0, w_down, ES, s.d, (uint64_t)s.E * s.f, KBLK, 128)) return MOE_ERR_CUDA;
      rc = launch<T, 256, DGRAD_DOWN, 2>(tA, tB0, tB0, p, pblocks * (s.f / 256), st);
    } else if (s.f % 256 == 0) {
      if (!make_tmap(&tB0, w_down, ES, s.d, (uint64_t)s.E * s.f, KBLK, 256)) return MOE_ERR_CUDA;
      rc = launch<T, 256, DGRAD_DOWN>(tA, tB0, tB0, p, mblocks * (s.f / 256), st);
    } else {
      if (!make_tmap(&tB0, w_down, ES, s.d, (uint64_t)s.E * s.f, KBLK, 128)) return MOE_ERR_CUDA;
      rc = launch<T, 128, DGRAD_DOWN>(tA, tB0, tB0, p, mblocks * (s.f / 128), st);
    }
    if (rc) return rc;
  }
  // (2) dWd[e] = a^T [f, rows_e] x dy_perm [rows_e, d]
  {
    // every expert's last partial K-block of a and dy_perm, zero past the expert's rows
    if (launch_wgrad_tails(a, s.f, tail_a, dy_perm, s.d, tail_b, offsets, s.E, st)) return MOE_ERR_CUDA;
    if (!make_tmap(&tAT, tail_a, ES, s.f, tail_rows, BOX_MN, KBLK) ||
        !make_tmap(&tBT, tail_b, ES, s.d, tail_rows, BOX_MN, KBLK))
      return MOE_ERR_CUDA;
    CUtensorMap tO;
    if (!make_tmap(&tO, dw_down, ES, s.d, (uint64_t)s.E * s.f, 64, 32)) return MOE_ERR_CUDA;
    if (!make_tmap(&tA, a, ES, s.f, P, BOX_MN, KBLK)) return MOE_ERR_CUDA;
    p.M = s.f; p.N = s.d; p.out0 = dw_down; p.aux = nullptr;
    if (s.d % 256 == 0 && s.f % 256 == 0) {
      // weight-gradient tiles are 256 weight rows (no empty rows): always CTA pairs
      if (!make_tmap(&tB0, dy_perm, ES, s.d, P, BOX_MN, KBLK)) return MOE_ERR_CUDA;
      rc = launch<T, 256, WGRAD_DOWN, 2>(tA, tB0, tB0, p, (int64_t)s.E * (s.f / 256) * (s.d / 256), st, &tO, &tO,
                                         &tAT, &tBT);
    } else if (s.d % 256 == 0) {
      if (!make_tmap(&tB0, dy_perm, ES, s.d, P, BOX_MN, KBLK)) return MOE_ERR_CUDA;
      rc = launch<T, 256, WGRAD_DOWN>(tA, tB0, tB0, p, (int64_t)s.E * (s.f / BM) * (s.d / 256), st, &tO, &tO, &tAT,
                                      &tBT);
    } else {
      if (!make_tmap(&tB0, dy_perm, ES, s.d, P, BOX_MN, KBLK)) return MOE_ERR_CUDA;
      rc = launch<T, 128, WGRAD_DOWN>(tA, tB0, tB0, p, (int64_t)s.E * (s.f / BM) * (s.d / 128), st, &tO, &tO, &tAT,
                                      &tBT);
    }
    if (rc) return rc;
  }
  // (3) dx_perm = dhu [P,2f] x [Wg | Wu]^T [2f,d]
  {
    if (!make_tmap(&tA, dhu, ES, 2 * s.f, P, KBLK, BM)) return MOE_ERR_CUDA;
    p.K = 2 * s.f; p.N = s.d; p.out0 = dx_perm;
    if (s.d % 256 == 0 && pair_rows(s)) {
      if (!make_tmap(&tB0, w_gate, ES, s.f, (uint64_t)s.E * s.d, KBLK, 128)) return MOE_ERR_CUDA;
      if (!make_tmap(&tB1, w_up, ES, s.f, (uint64_t)s.E * s.d, KBLK, 128)) return MOE_ERR_CUDA;
      rc = launch<T, 256, DGRAD_GU, 2>(tA, tB0, tB1, p, ((P + 255) / 256 + s.E) * (s.d / 256), st);
    } else if (s.d % 256 == 0) {
      if (!make_tmap(&tB0, w_gate, ES, s.f, (uint64_t)s.E * s.d, KBLK, 256)) return MOE_ERR_CUDA;
      if (!make_tmap(&tB1, w_up, ES, s.f, (uint64_t)s.E * s.d, KBLK, 256)) return MOE_ERR_CUDA;
      rc = launch<T, 256, DGRAD_GU>(tA, tB0, tB1, p, mblocks * (s.d / 256), st);
    } else {
      if (!make_tmap(&tB0, w_gate, ES, s.f, (uint64_t)s.E * s.d, KBLK, 128)) return MOE_ERR_CUDA;
      if (!make_tmap(&tB1, w_up, ES, s.f, (uint64_t)s.E * s.d, KBLK, 128)) return MOE_ERR_CUDA;
      rc = launch<T, 128, DGRAD_GU>(tA, tB0, tB1, p, mblocks * (s.d / 128), st);
    }
    if (rc) return rc;
  }
  // (4) [dWg | dWu][e] = x_perm^T [d, rows_e] x dhu [rows_e, 2f]
  {
    if (launch_wgrad_tails(x_perm, s.d, tail_a, dhu, 2 * s.f, tail_b, offsets, s.E, st)) return MOE_ERR_CUDA;
    if (!make_tmap(&tAT, tail_a, ES, s.d, tail_rows, BOX_MN, KBLK) ||
        !make_tmap(&tBT, tail_b, ES, 2 * s.f, tail_rows, BOX_MN, KBLK))
      return MOE_ERR_CUDA;
    if (!make_tmap(&tA, x_perm, ES, s.d, P, BOX_MN, KBLK)) return MOE_ERR_CUDA;
    if (!make_tmap(&tB0, dhu, ES, 2 * s.f, P, BOX_MN, KBLK)) return MOE_ERR_CUDA;
    CUtensorMap tO0, tO1;
    if (!make_tmap(&tO0, dw_gate, ES, s.f, (uint64_t)s.E * s.d, 64, 32) ||
        !make_tmap(&tO1, dw_up, ES, s.f, (uint64_t)s.E * s.d, 64, 32))
      return MOE_ERR_CUDA;
    p.M = s.d; p.N = 2 * s.f; p.out0 = dw_gate; p.out1 = dw_up;
    if (s.f % 256 == 0 && s.d % 256 == 0)
      rc = launch<T, 256, WGRAD_GU, 2>(tA, tB0, tB0, p, (int64_t)s.E * (s.d / 256) * (2 * s.f / 256), st, &tO0, &tO1,
                                       &tAT, &tBT);
    else if (s.f % 256 == 0)
      rc = launch<T, 256, WGRAD_GU>(tA, tB0, tB0, p, (int64_t)s.E * (s.d / BM) * (2 * s.f / 256), st, &tO0, &tO1,
                                    &tAT, &tBT);
    else
      rc = launch<T, 128, WGRAD_GU>(tA, tB0, tB0, p, (int64_t)s.E * (s.d / BM) * (2 * s.f / 128), st, &tO0, &tO1,
                                    &tAT, &tBT);
    if (rc) return rc;
  }
  return MOE_OK;
}

// Router on the tensor cores: logits = x [T,d] x W_r [d,E] (bf16 in, fp32 out) with the
// top-k and gates fused into the epilogue.  Needs E % 8 == 0 (16-byte TMA row pitch).
static int router_impl(const Shape &s, const void *x, const void *w_r, const float *bias, float *logits,
                       int32_t *idx, float *gate, int *err, cudaStream_t st) {
  constexpr int ES = 2, KBLK = 64, BOX_MN = 64;
  CUtensorMap tA, tB;
  if (!make_tmap(&tA, x, ES, s.d, s.T, KBLK, BM)) return MOE_ERR_CUDA;
  if (!make_tmap(&tB, w_r, ES, s.E, s.d, BOX_MN, KBLK)) return MOE_ERR_CUDA;
  Params p{};
  p.E = s.E; p.P = (int)s.T; p.K = s.d; p.d = s.d; p.f = s.f; p.k = s.k;
  p.out0 = idx; p.out1 = gate; p.out2 = logits; p.aux = bias; p.err = err; p.where = err + 1;
  const int64_t tiles = (s.T + BM - 1) / BM;
  const int bn = s.E <= 64 ? 64 : s.E <= 128 ? 128 : 256;
  p.N = bn;
  if (bn == 64) return launch<bf16, 64, ROUTER>(tA, tB, tB, p, tiles, st);
  if (bn == 128) return launch<bf16, 128, ROUTER>(tA, tB, tB, p, tiles, st);
  return launch<bf16, 256, ROUTER>(tA, tB, tB, p, tiles, st);
}

// ------------------------------------------------------------------ MXFP8 path
struct MxOp {
  uint8_t *codes, *scales;
};
static MxOp mx_r(void *ws, size_t off, int64_t rows, int64_t cols) {
  uint8_t *b = static_cast<uint8_t *>(ws) + off;
  return {b, b + rows * cols};
}

// Forward with both operands of both GEMMs quantised to MXFP8 (blocks along K).  Every
// quantiser writes its scales in the tile layout the GEMMs fetch with bulk copies.
static int mx_fwd_impl(const Shape &s, const void *x_perm, const int32_t *offsets, const void *w_gate,
                       const void *w_up, const void *w_down, void *hu, void *a, void *y_perm, void *ws,
                       cudaStream_t st, bool x_quantized, uint8_t *wsaved, bool wfill) {
  const WsLayout L = ws_layout(s);
  const int64_t P = s.P(), R = s.Ppad(), ed = (int64_t)s.E * s.d, ef = (int64_t)s.E * s.f;
  // x_perm's rows in MXFP8: in the caller's saved copies when given, else in the workspace
  const MxOp xq = wsaved ? mx_r(wsaved, mx_saved_layout(s).xq_r, R, s.d) : mx_r(ws, L.xq_r, R, s.d);
  const MxOp aq = mx_r(ws, L.aq_r, R, s.f);
  // x_quantized: the FP8 dispatch already wrote xq's rows
  if (!x_quantized && launch_mx_quant_rows(x_perm, P, s.d, offsets, s.E, R, xq.codes, xq.scales, st, true))
    return MOE_ERR_CUDA;
  MxOp wgu, wd;
  if (wsaved) {
    // the caller's buffer: every orientation from one read of each weight (wfill), or the
    // copies an earlier forward wrote there
    const MxSavedLayout M = mx_saved_layout(s);
    wgu = mx_r(wsaved, M.wgu_c, ed, 2 * s.f);
    wd = mx_r(wsaved, M.wd_c, ef, s.d);
    const MxOp wgur = mx_r(wsaved, M.wgu_r, ed, 2 * s.f), wdr = mx_r(wsaved, M.wd_r, ef, s.d);
    if (wfill && (launch_mx_quant_weights(w_gate, w_up, ed, s.f, true, wgu.codes, wgu.scales, wgur.codes,
                                          wgur.scales, st) ||
                  launch_mx_quant_weights(w_down, nullptr, ef, s.d, false, wd.codes, wd.scales, wdr.codes,
                                          wdr.scales, st)))
      return MOE_ERR_CUDA;
  } else {
    wgu = mx_r(ws, L.wgu_c, ed, 2 * s.f);
    wd = mx_r(ws, L.wd_c, ef, s.d);
    if (launch_mx_quant_cols_gu(w_gate, w_up, ed, s.f, wgu.codes, wgu.scales, st, true) ||
        (y_perm && launch_mx_quant_cols(w_down, ef, s.d, nullptr, s.E, ef, wd.codes, wd.scales, st, true)))
      return MOE_ERR_CUDA;
  }
  int *err = err_word(ws);
  Params p{};
  p.offsets = offsets; p.E = s.E; p.P = (int)P; p.f = s.f; p.d = s.d; p.err = err; p.where = err + 1;
  const int64_t mblocks = (P + BM - 1) / BM + s.E;
  CUtensorMap tA, tB;
  // GEMM 1: [h | u] tiles of 64 gate + 64 up columns
  if (!make_tmap(&tA, xq.codes, 1, s.d, R, 128, BM) || !make_tmap(&tB, wgu.codes, 1, 2 * s.f, ed, 128, 128))
    return MOE_ERR_CUDA;
  p.K = s.d; p.N = 2 * s.f; p.out0 = hu; p.out1 = a;
  p.sfa = xq.scales; p.nka = s.d / 128; p.sfb = wgu.scales; p.nkb = (int)(ed / 128);
  if (a && y_perm) {
    // the epilogue also writes a in MXFP8 along f, the down projection's operand, and (into
    // the caller's buffer, for the backward) down the padded token axis
    p.q_row_codes = aq.codes; p.q_row_scales = aq.scales; p.nk_row = s.f / 128;
    if (wsaved && wfill) {
      const MxOp aqt = mx_r(wsaved, mx_saved_layout(s).aq_t, R, s.f);
      p.q_col_codes = aqt.codes; p.q_col_scales = aqt.scales; p.nk_col = (int)((R + 127) / 128);
    }
  }
  int rc = launch<e4m3, 128, FWD_GU>(tA, tB, tB, p, mblocks * (p.N / 128), st);
  p.q_row_codes = p.q_row_scales = p.q_col_codes = p.q_col_scales = nullptr;
  if (rc || !y_perm) return rc;   // no y_perm: [h | u] only (the backward's recompute)
  // GEMM 2: y_perm = a Wd
  if (!make_tmap(&tA, aq.codes, 1, s.f, R, 128, BM) || !make_tmap(&tB, wd.codes, 1, s.d, ef, 128, 128))
    return MOE_ERR_CUDA;
  p.K = s.f; p.N = s.d; p.out0 = y_perm; p.out1 = nullptr;
  p.sfa = aq.scales; p.nka = s.f / 128; p.sfb = wd.scales; p.nkb = (int)(ef / 128);
  return launch<e4m3, 128, FWD_DOWN>(tA, tB, tB, p, mblocks * (p.N / 128), st);
}

// Backward with every GEMM operand quantised to MXFP8 along that GEMM's own K.
static int mx_bwd_impl(const Shape &s, const void *dy_perm, const void *x_perm, const void *hu, const void *a,
                       const int32_t *offsets, const void *w_gate, const void *w_up, const void *w_down, void *dhu,
                       void *dx_perm, void *dw_gate, void *dw_up, void *dw_down, void *ws, cudaStream_t st,
                       const uint8_t *wsaved, bool dy_quantized, bool keep_dhu) {
  const WsLayout L = ws_layout(s);
  const int64_t P = s.P(), R = s.Ppad(), ed = (int64_t)s.E * s.d, ef = (int64_t)s.E * s.f;
  const int nkt = (int)((R + 127) / 128);   // K groups of the token-axis operands
  const MxOp dyq = mx_r(ws, L.dyq_r, R, s.d), dhuq = mx_r(ws, L.dhuq_r, R, 2 * s.f);
  // the token-axis copies of x_perm and a: from the forward when it kept them
  uint8_t *wsv0 = const_cast<uint8_t *>(wsaved);
  const MxOp xqt = wsaved ? mx_r(wsv0, mx_saved_layout(s).xq_t, R, s.d) : mx_r(ws, L.xq_t, R, s.d);
  const MxOp aqt = wsaved ? mx_r(wsv0, mx_saved_layout(s).aq_t, R, s.f) : mx_r(ws, L.aq_t, R, s.f);
  const MxOp dyqt = mx_r(ws, L.dyq_t, R, s.d), dhuqt = mx_r(ws, L.dhuq_t, R, 2 * s.f);
  // the weights' data-gradient orientations: from the forward's copies when given
  const MxSavedLayout M = mx_saved_layout(s);
  uint8_t *wsv = const_cast<uint8_t *>(wsaved);
  const MxOp wdr = wsaved ? mx_r(wsv, M.wd_r, ef, s.d) : mx_r(ws, L.wd_r, ef, s.d);
  const MxOp wgur = wsaved ? mx_r(wsv, M.wgu_r, ed, 2 * s.f) : mx_r(ws, L.wgu_r, ed, 2 * s.f);
  int *err = err_word(ws);
  Params p{};
  p.offsets = offsets; p.E = s.E; p.P = (int)P; p.f = s.f; p.d = s.d; p.err = err; p.where = err + 1;
  const int64_t mblocks = (P + BM - 1) / BM + s.E;
  CUtensorMap tA, tB;
  int rc;
  // (1) da = dy Wd^T -> SwiGLU backward -> dhu
  // dy_quantized: the combine's backward already wrote dy_perm's codes in both orientations
  if ((!dy_quantized && launch_mx_quant_rows(dy_perm, P, s.d, offsets, s.E, R, dyq.codes, dyq.scales, st, true)) ||
      (!wsaved && launch_mx_quant_rows(w_down, ef, s.d, nullptr, s.E, ef, wdr.codes, wdr.scales, st, true)))
    return MOE_ERR_CUDA;
  if (!make_tmap(&tA, dyq.codes, 1, s.d, R, 128, BM) || !make_tmap(&tB, wdr.codes, 1, s.d, ef, 128, 128))
    return MOE_ERR_CUDA;
  // keep_dhu: [dh | du] in bf16 as well (nothing in the MXFP8 backward reads it)
  p.K = s.d; p.N = s.f; p.out0 = keep_dhu ? dhu : nullptr; p.aux = hu;
  p.sfa = dyq.scales; p.nka = s.d / 128; p.sfb = wdr.scales; p.nkb = s.d / 128;
  // the epilogue also writes [dh | du] in MXFP8 in both orientations the gate/up GEMMs read
  p.q_row_codes = dhuq.codes; p.q_row_scales = dhuq.scales; p.nk_row = 2 * s.f / 128;
  p.q_col_codes = dhuqt.codes; p.q_col_scales = dhuqt.scales; p.nk_col = nkt;
  rc = launch<e4m3, 128, DGRAD_DOWN>(tA, tB, tB, p, mblocks * (s.f / 128), st);
  p.q_row_codes = p.q_row_scales = p.q_col_codes = p.q_col_scales = nullptr;
  if (rc) return rc;
  // (2) dWd = a^T dy, K = the tokens of each expert
  if ((!wsaved && launch_mx_quant_cols(a, P, s.f, offsets, s.E, R, aqt.codes, aqt.scales, st, true)) ||
      (!dy_quantized && launch_mx_quant_cols(dy_perm, P, s.d, offsets, s.E, R, dyqt.codes, dyqt.scales, st, true)))
    return MOE_ERR_CUDA;
  if (!make_tmap(&tA, aqt.codes, 1, s.f, R, 128, 128) || !make_tmap(&tB, dyqt.codes, 1, s.d, R, 128, 128))
    return MOE_ERR_CUDA;
  CUtensorMap tO0, tO1;
  if (!make_tmap(&tO0, dw_down, 2, s.d, ef, 64, 32)) return MOE_ERR_CUDA;
  p.M = s.f; p.N = s.d; p.out0 = dw_down; p.aux = nullptr;
  p.sfa = aqt.scales; p.nka = nkt; p.sfb = dyqt.scales; p.nkb = nkt;
  rc = launch<e4m3, 128, WGRAD_DOWN>(tA, tB, tB, p, (int64_t)s.E * (s.f / BM) * (s.d / 128), st, &tO0, &tO0);
  if (rc) return rc;
  // (3) dx_perm = [dh | du] [Wg | Wu]^T
  if (!wsaved && launch_mx_quant_rows_gu(w_gate, w_up, ed, s.f, wgur.codes, wgur.scales, st, true))
    return MOE_ERR_CUDA;
  if (!make_tmap(&tA, dhuq.codes, 1, 2 * s.f, R, 128, BM) || !make_tmap(&tB, wgur.codes, 1, 2 * s.f, ed, 128, 128))
    return MOE_ERR_CUDA;
  p.K = 2 * s.f; p.N = s.d; p.out0 = dx_perm;
  p.sfa = dhuq.scales; p.nka = 2 * s.f / 128; p.sfb = wgur.scales; p.nkb = 2 * s.f / 128;
  rc = launch<e4m3, 128, DGRAD_GU>(tA, tB, tB, p, mblocks * (s.d / 128), st);
  if (rc) return rc;
  // (4) [dWg | dWu] = x^T [dh | du], K = the tokens of each expert
  if (!wsaved && launch_mx_quant_cols(x_perm, P, s.d, offsets, s.E, R, xqt.codes, xqt.scales, st, true))
    return MOE_ERR_CUDA;
  if (!make_tmap(&tA, xqt.codes, 1, s.d, R, 128, 128) || !make_tmap(&tB, dhuqt.codes, 1, 2 * s.f, R, 128, 128))
    return MOE_ERR_CUDA;
  if (!make_tmap(&tO0, dw_gate, 2, s.f, ed, 64, 32) || !make_tmap(&tO1, dw_up, 2, s.f, ed, 64, 32))
    return MOE_ERR_CUDA;
  p.M = s.d; p.N = 2 * s.f; p.out0 = dw_gate; p.out1 = dw_up;
  p.sfa = xqt.scales; p.nka = nkt; p.sfb = dhuqt.scales; p.nkb = nkt;
  return launch<e4m3, 128, WGRAD_GU>(tA, tB, tB, p, (int64_t)s.E * (s.d / BM) * (2 * s.f / 128), st, &tO0, &tO1);
}

}  // namespace gg

void set_gemm_stall_ns(uint64_t ns) { gg::g_stall_ns.store(ns, std::memory_order_relaxed); }

int launch_router_tc(const Shape &s, const void *x, const void *w_r, const float *bias, float *logits,
                     int32_t *idx, float *gate, int *err, cudaStream_t st) {
  return gg::router_impl(s, x, w_r, bias, logits, idx, gate, err, st);
}

int launch_grouped_fwd(const Shape &s, const void *x_perm, const int32_t *offsets, const void *w_gate,
                       const void *w_up, const void *w_down, void *hu, void *a, void *y_perm, void *ws,
                       cudaStream_t st, bool x_quantized, uint8_t *wsaved, bool wfill) {
  if (s.prec == MOE_PREC_MXFP8)
    return gg::mx_fwd_impl(s, x_perm, offsets, w_gate, w_up, w_down, hu, a, y_perm, ws, st, x_quantized, wsaved,
                           wfill);
  if (s.dtype == MOE_BF16)
    return gg::fwd_impl<bf16>(s, x_perm, offsets, w_gate, w_up, w_down, hu, a, y_perm, ws, st);
  return gg::fwd_impl<float>(s, x_perm, offsets, w_gate, w_up, w_down, hu, a, y_perm, ws, st);
}

int launch_grouped_bwd(const Shape &s, const void *dy_perm, const void *x_perm, const void *hu,
                       const void *a, const int32_t *offsets, const void *w_gate, const void *w_up,
                       const void *w_down, void *dhu, void *dx_perm, void *dw_gate, void *dw_up,
                       void *dw_down, void *ws, cudaStream_t st, const uint8_t *wsaved, bool dy_quantized,
                       bool keep_dhu) {
  // The weight-gradient GEMMs reduce over tokens, which makes both operands MN-major;
  // tf32 MMAs take K-major operands only, so the fp32 backward is not offered.
  if (s.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (s.prec == MOE_PREC_MXFP8)
    return gg::mx_bwd_impl(s, dy_perm, x_perm, hu, a, offsets, w_gate, w_up, w_down, dhu, dx_perm, dw_gate,
                           dw_up, dw_down, ws, st, wsaved, dy_quantized, keep_dhu);
  return gg::bwd_impl<bf16>(s, dy_perm, x_perm, hu, a, offsets, w_gate, w_up, w_down, dhu, dx_perm,
                            dw_gate, dw_up, dw_down, ws, st);
}

}  // namespace moe
