// moe_build_offsets_noalloc: the routing-metadata step for callers that cannot allocate.
//
// moe_build_offsets needs a caller-provided workspace for its per-block expert
// histograms.  Some callers have no way to provide one: a host program that hands all of
// the GPU's memory to its own pool at start-up (so an extra cudaMalloc fails or fragments
// that pool), or a C caller whose interface passes only the routing tensors and has no
// allocator of its own to make a scratch buffer with.  For them this entry point keeps
// its scratch in a fixed array that is part of the library image itself.
#include <mutex>

#include "common.cuh"

namespace {

// Per-block histograms of the metadata kernels: ceil(T*k / 1024) * E int32 entries.
constexpr size_t NOALLOC_SCRATCH_INTS = 65536;  // 256 KiB

// Lives in device memory on every GPU that loads this library, until the process exits.
// Every call uses the same array, so calls whose work overlaps on the GPU (two streams,
// or two host threads) race on it; the caller must order them.
static __device__ __align__(256) int32_t g_noalloc_scratch[NOALLOC_SCRATCH_INTS];

constexpr int MAX_DEVICES = 64;
std::mutex g_mu;
void *g_scratch_ptr[MAX_DEVICES] = {};

// The array's name in host code is only a host-side handle, not a device address: the
// kernels must be given the address cudaGetSymbolAddress returns for the current device.
// Resolved once per device, on the first call made with that device current, in the context
// current then (the primary context, for callers of the runtime API); the address is only
// valid in that context.
int scratch_for_current_device(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" int moe_build_offsets_noalloc(const moe_config *cfg, const int32_t *topk_idx, int32_t *counts,
                                         int32_t *offsets, int32_t *slot_of_pair, int32_t *pair_of_slot,
                                         moe_stream_t stream) {
  if (!cfg || cfg->T < 0 || cfg->E <= 0 || cfg->k <= 0 || cfg->d <= 0 || cfg->f <= 0)
    return MOE_ERR_INVALID_ARG;
  if (cfg->E > moe::MAX_E || cfg->k > moe::MAX_K || cfg->k > cfg->E) return MOE_ERR_UNSUPPORTED;
  if (cfg->T * (int64_t)cfg->k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!topk_idx || !slot_of_pair || !pair_of_slot)) return MOE_ERR_INVALID_ARG;
  moe::Shape s = moe::shape_of(cfg);
  const int64_t nblocks = (s.P() + moe::SCATTER_CHUNK - 1) / moe::SCATTER_CHUNK;
  if ((uint64_t)nblocks * (uint64_t)s.E > NOALLOC_SCRATCH_INTS) return MOE_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  int rc = scratch_for_current_device(&scratch);
  if (rc) return rc;
  // The histogram kernel overwrites every entry it later reads, so nothing needs clearing.
  // No error word: an expert index outside [0, E) leaves the outputs undefined, unreported.
  cudaError_t e = moe::launch_build_offsets(s, topk_idx, counts, offsets, slot_of_pair, pair_of_slot,
                                            static_cast<int32_t *>(scratch), nullptr,
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
